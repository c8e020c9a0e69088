// attn_simt.cu -- split-context paged attention on CUDA cores, for row
// blocks of four query rows: head dim 512 calls with up to four rows per KV
// head (decode at GQA <= 4), and every call whose page size is not a
// multiple of 128 (the tensor-core kernels' tiles stay inside a page).
//
// TensorFold #1620 ("Kolibri-1's full layers take their K/V from pages of
// the core pool"): decode reads keys through the page table, split across
// the context (the partial kernel) and merged (the merge kernel, which reads
// no pages); its later comment moves the page lookup out of the per-key loop
// to once per tile.  Here each page id is read once, one page before its
// first tile is needed.
//
// Layout of one CTA (persistent, one per SM):
//   last warp     producer (one lane): walks the CTA's segments one segment
//                 ahead; per segment it copies the four query rows into a
//                 double-buffered shared slot and streams K and V tiles of TK
//                 positions into a ring of NSTAGE stages with bulk copies
//                 (TMA engine, no tensor map: a tile of one page and KV head
//                 is one contiguous run).  With a page size that is not a
//                 multiple of TK a tile may straddle pages: tiles are then
//                 armed four at a time (a quad of contiguous stages, complete
//                 on one barrier) and one copy covers a page's run across
//                 them.  Page ids are read one page early.
//   other warps   consumers: tile T of the CTA's sequence goes to consumer
//                 warp T % NCW.  A warp keeps its own online-softmax state
//                 (running max m, running sum l, unnormalised O) for the four
//                 rows of the segment.  At the end of the segment each warp parks
//                 its state in shared memory; the last warp to arrive
//                 combines them and writes the segment's result (the normalised
//                 output when the row block has one chunk, else a partial for
//                 the merge kernel).  No CTA-wide barrier: the other warps go
//                 straight on to the next segment.
//
// Inner loop of a consumer warp on one tile (head dim 128, TK = 32):
//   scores  the warp is 4 groups of 8 lanes; group g takes 8 keys, lane i of
//           a group holds 16 of the 128 dims of the 4 query rows as packed
//           bf16 pairs and accumulates 8 keys x 4 rows partial dots with
//           bf16 x bf16 -> fp32 FMAs (fma.rn.f32.bf16: exact products, fp32
//           sums, no conversions); three butterfly rounds (reduce-scatter
//           over the 8 lanes) leave lane L with the 4 rows' full scores of
//           key L.
//   softmax tile max per row by warp shuffles, exp2 of log2-scaled scores;
//           masked positions are SELECTED to -inf (never multiplied), so NaN
//           in unused slots cannot leak.  A causal row sees positions below
//           its limit; under tree masks (kTree) a row sees the positions
//           before the window and the window rows its mask byte names.
//   PV      lane L owns dims 4L..4L+3 of the 4 output rows as fp32 pairs and
//           updates them with packed fp32 FMAs (two per instruction);
//           probabilities come from a per-warp shared buffer; only positions
//           below the segment's end are visited, so no unused slot is read.
// Head dim 512 uses TK = 8 and one group of 32 lanes; the same steps.
#include "launch.cuh"
#include "plan.cuh"

namespace tfp {

template <int D>
struct SimtCfg;
// Registers are split per SM sub-partition: with 9 warps one sub-partition
// holds 3 warps (at most 168 registers each), with 8 warps 2 (255 each).
// Seven consumers (8 warps with the producer) measured faster than eight at
// head dim 128: decode 12 x 40,960 in pages of 37 3,745 against 3,442 GB/s,
// 64 x 2,048 5,576 against 5,160 -- the producer lane no longer shares a
// sub-partition with two busy consumer warps.
template <>
struct SimtCfg<128> {
    static constexpr int TK = 32;      // positions per tile
    static constexpr int LG = 8;       // lanes sharing one key's dot product
    static constexpr int NSTAGE = 12;  // ring depth (16 KB per stage)
    static constexpr int NCW = 7;      // consumer warps
};
template <>
struct SimtCfg<512> {
    static constexpr int TK = 8;
    static constexpr int LG = 32;
    static constexpr int NSTAGE = 8;
    static constexpr int NCW = 7;
};

constexpr int kR = kSimtRows;  // query rows per row block
template <int D>
constexpr int simt_threads() { return 32 * (SimtCfg<D>::NCW + 1); }

template <int D>
struct SimtSmem {
    static constexpr int TK = SimtCfg<D>::TK;
    static constexpr int NSTAGE = SimtCfg<D>::NSTAGE;
    static constexpr int NCW = SimtCfg<D>::NCW;
    static constexpr int TILE_BYTES = TK * D * 2;
    // K and V rings: consecutive stages are contiguous, so a copy of a page
    // piece may run across the stages of one quad (below)
    alignas(128) uint8_t kring[NSTAGE][TILE_BYTES];
    alignas(128) uint8_t vring[NSTAGE][TILE_BYTES];
    alignas(16) __nv_bfloat16 qbuf[2][kR][D];      // the segment's query rows (double buffer)
    alignas(16) float pbuf[NCW][TK][2 * kR];        // per key: p0,p0,p1,p1,p2,p2,p3,p3
    alignas(16) float wo[NCW][kR][D];               // parked warp states
    float wm[NCW][kR];
    float wl[NCW][kR];
    uint64_t full[NSTAGE];
    uint64_t empty[NSTAGE];
    // Tile each stage was last armed for.  Consumers take tiles round-robin
    // and the ring is deeper than the number of consumers, so a warp can
    // reach stage s for tile T while the stage's previous tile (T - NSTAGE,
    // another warp's) is still in flight; a parity wait alone cannot tell
    // those phases apart.  The tag can: it moves to T only after tile
    // T - NSTAGE has been consumed.
    volatile uint32_t stage_tile[NSTAGE];
    uint64_t q_full[2];
    uint64_t q_empty[2];
    uint64_t w_free;       // the parked-state slot is free again (combine done)
    int w_count;           // warps parked for the current segment
    CtaRange range;        // this CTA's tiles
    volatile int abort_flag;
    long long wait_limit;  // cycles a pipeline wait may take (the call's)
};

template <int D>
size_t simt_smem_bytes()
{
    return sizeof(SimtSmem<D>);
}

__device__ __forceinline__ float warp_max(float v, int lo_mask)
{
#pragma unroll
    for (int m = 16; m >= lo_mask; m >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
    return v;
}

__device__ __forceinline__ float warp_sum(float v, int lo_mask)
{
#pragma unroll
    for (int m = 16; m >= lo_mask; m >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

// c + a.lo * b.lo + a.hi * b.hi for two packed bf16 pairs; each step is one
// fp32 FMA of an exact bf16 x bf16 product.
__device__ __forceinline__ float fma_bf16x2(uint32_t a, uint32_t b, float c)
{
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "+f"(c)
        : "r"(a), "r"(b));
    return c;
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) { return make_float2(bf_lo(w), bf_hi(w)); }

// A bounded wait that turns a timeout into the abort state of the CTA.
template <int D>
__device__ __forceinline__ bool wait_or_abort(SimtSmem<D> &sm, uint64_t *bar, uint32_t parity,
                                              uint32_t *flags, uint32_t site)
{
    if (sm.abort_flag)
        return false;
    if (mbar_wait(bar, parity, sm.wait_limit))
        return true;
    set_flag(flags, kDevTimeout);
    set_flag(flags + 1, site);
    sm.abort_flag = 1;
    return false;
}

// Waits until stage `stage` has been armed for tile T (bounded like the
// mbarrier waits); after that its full barrier's parity refers to tile T.
template <int D>
__device__ __forceinline__ bool wait_tag(SimtSmem<D> &sm, int stage, uint32_t T, uint32_t *flags)
{
    if (sm.stage_tile[stage] == T)
        return true;
    const long long t0 = clock64();
    while (sm.stage_tile[stage] != T) {
        if (sm.abort_flag)
            return false;
        if (clock64() - t0 > sm.wait_limit) {
            set_flag(flags, kDevTimeout);
            set_flag(flags + 1, kWaitTag);
            sm.abort_flag = 1;
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// Adds `bytes` to the transaction count of the barrier's current phase (no
// arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Copies the four query rows of segment `it` into q slot (j & 1).
template <int D>
__device__ __forceinline__ bool producer_q(const AttnParams &p, SimtSmem<D> &sm,
                                           const WorkItem &it, uint32_t j, uint64_t pol)
{
    const int slot = j & 1;
    if (!wait_or_abort(sm, &sm.q_empty[slot], ((j >> 1) & 1u) ^ 1u, p.flags, kWaitQEmpty))
        return false;
    mbar_arrive_expect_tx(&sm.q_full[slot], kR * D * 2);
    for (int r = 0; r < kR; ++r) {
        const int mm = min(it.b * kR + r, p.M - 1);
        const int wr = mm / p.G;
        const int h = it.kh * p.G + (mm - wr * p.G);
        bulk_g2s(sm.qbuf[slot][r], p.q + (((size_t)it.s * p.W + wr) * p.Hq + h) * D, D * 2,
                 &sm.q_full[slot], pol);
    }
    return true;
}

// One lane.  Looks one segment ahead: the next segment's query rows are copied
// when the current segment starts, and every page id is read one page before
// its first tile, so no table read sits on the copy path.
template <int D>
__device__ __forceinline__ void simt_producer(const AttnParams &p, SimtSmem<D> &sm)
{
    constexpr int TK = SimtCfg<D>::TK;
    constexpr int NSTAGE = SimtCfg<D>::NSTAGE;
    const uint64_t pol = l2_evict_first_policy();
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it, nx;
    uint32_t T = 0;
    uint32_t j = 0;  // segment counter of this CTA
    uint32_t q_issued = 0;  // segments whose query copy was started
    bool have = cur.next(p, it);
    if (have && producer_q<D>(p, sm, it, 0, pol))
        q_issued = 1;
    int32_t page_next = have ? __ldg(p.table + (int64_t)it.s * p.table_stride + it.key0 / p.P) : 0;
    // tiles assembled from page pieces: the quad being armed and the pending
    // copy (pc_n positions of page pc_page, KV head pc_kh, from offset pc_off,
    // into ring rows from pc_row)
    const bool quads = p.P % TK != 0;
    static_assert(NSTAGE % 4 == 0, "quads of stages");
    int quad = -1;
    int pc_n = 0, pc_pos = 0, pc_row = 0, pc_kh = 0, pc_off = 0;
    int32_t pc_page = 0;
    auto flush = [&]() {
        if (pc_n == 0)
            return;
        uint64_t *bar = &sm.full[(quad * 4 + 3) % NSTAGE];
        const uint32_t nb = static_cast<uint32_t>(pc_n) * D * 2u;
        if (pc_page >= 0 && pc_page < p.n_pages) {
            const size_t off = (((size_t)pc_page * p.Hkv + pc_kh) * p.P + pc_off) * D;
            mbar_expect_tx(bar, 2u * nb);
            bulk_g2s(&sm.kring[0][0] + (size_t)pc_row * D * 2, p.k_pool + off, nb, bar, pol);
            bulk_g2s(&sm.vring[0][0] + (size_t)pc_row * D * 2, p.v_pool + off, nb, bar, pol);
        } else {
            set_flag(p.flags, kDevBadPage);
        }
        pc_n = 0;
    };
    while (have && !sm.abort_flag) {
        SegCursor ahead = cur;
        const bool have_nx = ahead.next(p, nx);
        if (have_nx && producer_q<D>(p, sm, nx, j + 1, pol))
            q_issued = j + 2;
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        if (quads) {
            // Any page size: a tile of TK positions may straddle pages.  The
            // copy engine's cost is per copy (about 5 million copies a second
            // per SM, whatever their size up to a tile), so tiles are armed
            // four at a time: the quad's stages are contiguous in each ring,
            // and one bulk copy covers a page's run of positions across them
            // (pages of 37: about 1.1 copies per 32 positions instead of
            // 1.9).  Each copy adds its bytes to the quad's barrier (that of
            // its last stage), and the quad's one arrival closes it.  The
            // page walk moves forward piece by piece; the next page id is read
            // one page ahead.  A piece on a page outside the pool is not read
            // (and flagged).
            int lp = it.key0 / p.P;
            int page_end = (lp + 1) * p.P;
            int32_t page = __ldg(trow + lp);
            int32_t page_nx = page_end < it.key1 ? __ldg(trow + lp + 1) : 0;
            for (int t0 = it.key0; t0 < it.key1 && !sm.abort_flag; t0 += TK, ++T) {
                const int stage = T % NSTAGE;
                if ((int)(T >> 2) != quad) {
                    if (quad >= 0) {
                        flush();
                        mbar_arrive(&sm.full[(quad * 4 + 3) % NSTAGE]);
                    }
                    quad = (int)(T >> 2);
                }
                if (!wait_or_abort(sm, &sm.empty[stage], ((T / NSTAGE) & 1u) ^ 1u, p.flags, kWaitEmpty))
                    break;
                sm.stage_tile[stage] = T;
                const int t1 = min(t0 + TK, it.key1);
                for (int pos = t0; pos < t1;) {
                    const int n = min(page_end, t1) - pos;
                    const int row = stage * TK + (pos - t0);
                    // the pending run goes on if the source rows and the ring
                    // rows both continue it
                    if (pc_n > 0 && pc_page == page && pc_kh == it.kh && pc_pos + pc_n == pos &&
                        pc_row + pc_n == row) {
                        pc_n += n;
                    } else {
                        flush();
                        pc_n = n;
                        pc_pos = pos;
                        pc_row = row;
                        pc_page = page;
                        pc_kh = it.kh;
                        pc_off = pos - (page_end - p.P);
                    }
                    pos += n;
                    if (pos == page_end) {
                        ++lp;
                        page_end += p.P;
                        page = page_nx;
                        if (page_end < it.key1)   // page lp + 1 holds keys of this segment
                            page_nx = __ldg(trow + lp + 1);
                    }
                }
            }
            // The segment's last quad closes here and the next segment starts
            // a quad of its own: a quad never waits on a later segment, so no
            // consumer can be held on a tile whose quad the producer closes
            // only after a wait (the next query copy) that needs that
            // consumer.  The skipped slots keep their empty barriers' phases
            // in step: the producer releases them itself.  It first waits for
            // their previous tiles' releases and only then closes the quad: a
            // quad closes once every consumer of its slots' previous round is
            // past its wait on the quad's barrier, or that barrier could move
            // a phase further before such a consumer looks at it.
            const uint32_t T_end = T;
            bool skipped_ok = true;
            for (uint32_t Ts = T_end; (Ts & 3u) != 0u; ++Ts) {
                const int stage = Ts % NSTAGE;
                skipped_ok = skipped_ok && wait_or_abort(sm, &sm.empty[stage],
                                                         ((Ts / NSTAGE) & 1u) ^ 1u, p.flags, kWaitEmpty);
            }
            if (quad >= 0) {
                flush();
                mbar_arrive(&sm.full[(quad * 4 + 3) % NSTAGE]);
                quad = -1;
            }
            for (; (T & 3u) != 0u; ++T) {
                if (skipped_ok)
                    mbar_arrive(&sm.empty[T % NSTAGE]);
            }
            have = have_nx;
            it = nx;
            cur = ahead;
            ++j;
            continue;
        }
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
            const size_t base = (((size_t)(page_ok ? page : 0) * p.Hkv + it.kh) * p.P) * D;
            for (int t0 = pos0; t0 < pos1; t0 += TK, ++T) {
                const int stage = T % NSTAGE;
                if (!wait_or_abort(sm, &sm.empty[stage], ((T / NSTAGE) & 1u) ^ 1u, p.flags, kWaitEmpty))
                    break;
                sm.stage_tile[stage] = T;
                const int nk = min(TK, pos1 - t0);
                const uint32_t bytes = static_cast<uint32_t>(nk) * D * 2u;
                if (page_ok) {
                    const size_t off = base + (size_t)(t0 - lp * p.P) * D;
                    mbar_arrive_expect_tx(&sm.full[stage], 2u * bytes);
                    bulk_g2s(sm.kring[stage], p.k_pool + off, bytes, &sm.full[stage], pol);
                    bulk_g2s(sm.vring[stage], p.v_pool + off, bytes, &sm.full[stage], pol);
                } else {
                    mbar_arrive(&sm.full[stage]);
                }
            }
        }
        have = have_nx;
        it = nx;
        cur = ahead;
        ++j;
    }
    {
        // Let every copy this CTA started land before the CTA can exit.  On
        // the normal path every tile and query copy was consumed and these
        // phases are complete; after a consumer gave up, some may not be.
        const uint32_t n = T < (uint32_t)NSTAGE ? T : (uint32_t)NSTAGE;
        for (uint32_t k = 1; k <= n; ++k) {
            const uint32_t t = T - k;
            // (quads complete on the barrier of their last stage)
            const uint32_t b = quads ? ((t | 3u) % NSTAGE) : (t % NSTAGE);
            (void)mbar_wait(&sm.full[b], (t / NSTAGE) & 1u, sm.wait_limit);
        }
        for (uint32_t k = 1; k <= 2 && k <= q_issued; ++k) {
            const uint32_t jj = q_issued - k;  // the last two query copies started
            (void)mbar_wait(&sm.q_full[jj & 1], (jj >> 1) & 1u, sm.wait_limit);
        }
    }
}

// Tree masks (kTree): row r sees the positions before the window (pos <
// lim[r] = len - W) and window row c when bit c of tm[r] is set.
template <bool kTree>
__device__ __forceinline__ bool simt_sees(int pos, int lim, uint32_t tm, int base, int W)
{
    if constexpr (kTree)
        return pos < lim || ((unsigned)(pos - base) < (unsigned)W && ((tm >> (pos - base)) & 1u));
    else
        return pos < lim;
}

template <int D, bool kTree>
__device__ __forceinline__ void simt_consumer(const AttnParams &p, SimtSmem<D> &sm, int warp,
                                              int lane)
{
    constexpr int TK = SimtCfg<D>::TK;
    constexpr int NSTAGE = SimtCfg<D>::NSTAGE;
    constexpr int LG = SimtCfg<D>::LG;
    constexpr int NCW = SimtCfg<D>::NCW;
    constexpr int NG = 32 / LG;        // key groups per warp
    constexpr int KPG = TK / NG;       // keys per group
    constexpr int NACC = KPG * kR;     // partial dots per lane
    constexpr int NV = NACC / LG;      // full scores per lane after the reduce-scatter
    constexpr int CPL = D / 8 / LG;    // 16-byte chunks of a key row per lane
    constexpr int DL = D / 32;         // output dims per lane
    constexpr int LOG_LG = (LG == 8) ? 3 : 5;
    static_assert((1 << LOG_LG) == LG, "lane group");
    static_assert(NACC == 32 && CPL == 2, "tile shape");
    static_assert(NV == kR || NV == 1, "score ownership");

    const int grp = lane / LG;
    const int li = lane % LG;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const bool quads = p.P % TK != 0;

    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t T0 = 0;  // CTA tile index of the segment's first tile
    uint32_t j = 0;

    for (; cur.next(p, it); ++j) {
        // --- this segment's query rows: packed bf16 pairs in registers --------
        uint32_t qh[kR][CPL * 4];
        int lim[kR];
        uint32_t tm[kR];
        const int base = it.len - p.W;  // the window's first position
        {
            const int slot = j & 1;
            const bool ok = wait_or_abort(sm, &sm.q_full[slot], (j >> 1) & 1u, p.flags, kWaitQFull);
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                const int m = it.b * kR + r;
                if constexpr (kTree) {
                    lim[r] = base;
                    tm[r] = m < p.M ? __ldg(p.tree + (size_t)it.s * p.W + m / p.G) : 0u;
                } else {
                    lim[r] = row_lim(p, it.len, m);
                    tm[r] = 0u;
                }
                const bool live = ok && m < p.M;
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const uint4 w =
                        *reinterpret_cast<const uint4 *>(&sm.qbuf[slot][r][(li + c * LG) * 8]);
                    qh[r][c * 4 + 0] = live ? w.x : 0u;
                    qh[r][c * 4 + 1] = live ? w.y : 0u;
                    qh[r][c * 4 + 2] = live ? w.z : 0u;
                    qh[r][c * 4 + 3] = live ? w.w : 0u;
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.q_empty[slot]);
        }

        float m_run[kR], l_lane[NV];
        float2 o2[kR][DL / 2];
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            m_run[r] = NEG_INF;
#pragma unroll
            for (int e = 0; e < DL / 2; ++e)
                o2[r][e] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int jj = 0; jj < NV; ++jj)
            l_lane[jj] = 0.f;

        const int ntiles = (it.key1 - it.key0 + TK - 1) / TK;
        int t = (warp - (int)(T0 % NCW) + NCW) % NCW;
        for (; t < ntiles; t += NCW) {
            const uint32_t T = T0 + t;
            const int stage = T % NSTAGE;
            // the warp takes one decision: a lane whose wait ran out makes
            // every lane skip the tile (the CTA is winding down then)
            // (tiles assembled from page pieces complete per quad of stages)
            const int fs = quads ? (stage | 3) : stage;
            const bool ok = __all_sync(
                0xffffffffu, wait_tag<D>(sm, stage, T, p.flags) &&
                                 wait_or_abort(sm, &sm.full[fs], (T / NSTAGE) & 1u, p.flags,
                                               kWaitFull));
            if (!ok)
                continue;
            const uint8_t *Ks = sm.kring[stage];
            const uint8_t *Vs = sm.vring[stage];
            const int tpos = it.key0 + t * TK;
            const int nk = min(TK, it.key1 - tpos);

            // --- partial dot products: 8 keys x 4 rows over this lane's dims
            float acc[NACC];
#pragma unroll
            for (int x = 0; x < NACC; ++x)
                acc[x] = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int chunk = li + c * LG;
#pragma unroll
                for (int kk = 0; kk < KPG; ++kk) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(
                        Ks + (grp * KPG + kk) * D * 2 + chunk * 16);
#pragma unroll
                    for (int r = 0; r < kR; ++r) {
                        float a = acc[kk * kR + r];
                        a = fma_bf16x2(qh[r][c * 4 + 0], w.x, a);
                        a = fma_bf16x2(qh[r][c * 4 + 1], w.y, a);
                        a = fma_bf16x2(qh[r][c * 4 + 2], w.z, a);
                        a = fma_bf16x2(qh[r][c * 4 + 3], w.w, a);
                        acc[kk * kR + r] = a;
                    }
                }
            }
            // --- reduce-scatter over the LG lanes of the group -------------
            // Round with mask msk keeps the upper half of the array in lanes
            // whose bit msk is set.  Afterwards lane li holds entries
            // x = li * NV + j (j < NV) of the original kk * kR + r numbering.
#pragma unroll
            for (int rnd = 0; rnd < LOG_LG; ++rnd) {
                const int msk = LG >> (rnd + 1);
                const int half = NACC >> (rnd + 1);
                const bool upper = (li & msk) != 0;
#pragma unroll
                for (int x = 0; x < half; ++x) {
                    const float send = upper ? acc[x] : acc[x + half];
                    const float keep = upper ? acc[x + half] : acc[x];
                    acc[x] = keep + __shfl_xor_sync(0xffffffffu, send, msk);
                }
            }

            // --- masked log2-scaled scores, tile max, online softmax -------
            float sc[NV];
            float tmax[kR];
            if constexpr (NV == kR) {
                const int key = grp * KPG + li;  // == lane
                const int pos = tpos + key;
#pragma unroll
                for (int r = 0; r < kR; ++r) {
                    const bool vis = key < nk && simt_sees<kTree>(pos, lim[r], tm[r], base, p.W);
                    sc[r] = vis ? acc[r] * p.scale_log2 : NEG_INF;
                    tmax[r] = warp_max(sc[r], 1);
                }
            } else {
                const int key = li >> 2;
                const int r = li & 3;
                const int pos = tpos + key;
                const int my_lim = r == 0 ? lim[0] : r == 1 ? lim[1] : r == 2 ? lim[2] : lim[3];
                const uint32_t my_tm = r == 0 ? tm[0] : r == 1 ? tm[1] : r == 2 ? tm[2] : tm[3];
                const bool vis = key < nk && simt_sees<kTree>(pos, my_lim, my_tm, base, p.W);
                sc[0] = vis ? acc[0] * p.scale_log2 : NEG_INF;
                const float rm = warp_max(sc[0], 4);  // over the lanes of this row
#pragma unroll
                for (int rr = 0; rr < kR; ++rr)
                    tmax[rr] = __shfl_sync(0xffffffffu, rm, rr);
            }
            float m_use[kR], alpha[kR];
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                const float mn = fmaxf(m_run[r], tmax[r]);
                m_use[r] = mn == NEG_INF ? 0.f : mn;
                alpha[r] = fast_exp2(m_run[r] - m_use[r]);
                m_run[r] = mn;
            }
            float *pb = &sm.pbuf[warp][0][0];
            if constexpr (NV == kR) {
                float pr[kR];
#pragma unroll
                for (int r = 0; r < kR; ++r) {
                    pr[r] = fast_exp2(sc[r] - m_use[r]);
                    l_lane[r] = fmaf(l_lane[r], alpha[r], pr[r]);
                }
                float4 *dst = reinterpret_cast<float4 *>(pb + lane * 2 * kR);
                dst[0] = make_float4(pr[0], pr[0], pr[1], pr[1]);
                dst[1] = make_float4(pr[2], pr[2], pr[3], pr[3]);
            } else {
                const int r = li & 3;
                const float mu = r == 0 ? m_use[0] : r == 1 ? m_use[1] : r == 2 ? m_use[2] : m_use[3];
                const float al = r == 0 ? alpha[0] : r == 1 ? alpha[1] : r == 2 ? alpha[2] : alpha[3];
                const float pr = fast_exp2(sc[0] - mu);
                l_lane[0] = fmaf(l_lane[0], al, pr);
                *reinterpret_cast<float2 *>(pb + lane * 2) = make_float2(pr, pr);
            }
            __syncwarp();

            // --- O = alpha * O + P V over the visited positions -----------
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                const float2 a2 = make_float2(alpha[r], alpha[r]);
#pragma unroll
                for (int e = 0; e < DL / 2; ++e)
                    o2[r][e] = __fmul2_rn(o2[r][e], a2);
            }

            auto pv_step = [&](int kk) {
                const float4 pa = *reinterpret_cast<const float4 *>(pb + kk * 2 * kR);
                const float4 pc = *reinterpret_cast<const float4 *>(pb + kk * 2 * kR + 4);
                const float2 pr[4] = {make_float2(pa.x, pa.y), make_float2(pa.z, pa.w),
                                      make_float2(pc.x, pc.y), make_float2(pc.z, pc.w)};
                if constexpr (D == 128) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(Vs + kk * D * 2 + lane * 8);
                    const float2 v01 = bf2_to_f2(w.x), v23 = bf2_to_f2(w.y);
#pragma unroll
                    for (int r = 0; r < kR; ++r) {
                        o2[r][0] = __ffma2_rn(pr[r], v01, o2[r][0]);
                        o2[r][1] = __ffma2_rn(pr[r], v23, o2[r][1]);
                    }
                } else {
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(Vs + kk * D * 2 + lane * 16);
                    const uint4 w1 =
                        *reinterpret_cast<const uint4 *>(Vs + kk * D * 2 + D + lane * 16);
                    const float2 v[8] = {bf2_to_f2(w0.x), bf2_to_f2(w0.y), bf2_to_f2(w0.z),
                                         bf2_to_f2(w0.w), bf2_to_f2(w1.x), bf2_to_f2(w1.y),
                                         bf2_to_f2(w1.z), bf2_to_f2(w1.w)};
#pragma unroll
                    for (int r = 0; r < kR; ++r)
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            o2[r][e] = __ffma2_rn(pr[r], v[e], o2[r][e]);
                }
            };
            if (nk == TK) {
#pragma unroll
                for (int kk = 0; kk < TK; ++kk)
                    pv_step(kk);
            } else {
#pragma unroll 1
                for (int kk = 0; kk < nk; ++kk)
                    pv_step(kk);
            }
            __syncwarp();
            // (the test switch: every CTA withholds the release of its first tile)
            if (lane == 0 && !(p.withhold && T == 0))
                mbar_arrive(&sm.empty[stage]);
        }
        T0 += ntiles;
        if (quads)  // each segment's tiles start a quad (as the producer arms them)
            T0 = (T0 + 3u) & ~3u;

        // --- park this warp's state; the last warp in combines -------------
        float l_row[kR];
        if constexpr (NV == kR) {
#pragma unroll
            for (int r = 0; r < kR; ++r)
                l_row[r] = warp_sum(l_lane[r], 1);
        } else {
            const float lr = warp_sum(l_lane[0], 4);
#pragma unroll
            for (int r = 0; r < kR; ++r)
                l_row[r] = __shfl_sync(0xffffffffu, lr, r);
        }
        // the slot is free once the previous segment's combine is done
        (void)wait_or_abort(sm, &sm.w_free, (j & 1u) ^ 1u, p.flags, kWaitFree);
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                sm.wm[warp][r] = m_run[r];
                sm.wl[warp][r] = l_row[r];
            }
        }
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            if constexpr (D == 128) {
                *reinterpret_cast<float4 *>(&sm.wo[warp][r][lane * 4]) =
                    make_float4(o2[r][0].x, o2[r][0].y, o2[r][1].x, o2[r][1].y);
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    *reinterpret_cast<float4 *>(&sm.wo[warp][r][h * 256 + lane * 8]) =
                        make_float4(o2[r][h * 4 + 0].x, o2[r][h * 4 + 0].y, o2[r][h * 4 + 1].x,
                                    o2[r][h * 4 + 1].y);
                    *reinterpret_cast<float4 *>(&sm.wo[warp][r][h * 256 + lane * 8 + 4]) =
                        make_float4(o2[r][h * 4 + 2].x, o2[r][h * 4 + 2].y, o2[r][h * 4 + 3].x,
                                    o2[r][h * 4 + 3].y);
                }
            }
        }
        __syncwarp();
        int arrived = 0;
        if (lane == 0) {
            __threadfence_block();
            arrived = atomicAdd(&sm.w_count, 1);
        }
        arrived = __shfl_sync(0xffffffffu, arrived, 0);
        if (arrived != NCW - 1)
            continue;

        // --- this warp is the last one in: combine the NCW states ----------
        if (lane == 0)
            sm.w_count = 0;
        __threadfence_block();
#pragma unroll 1
        for (int r = 0; r < kR; ++r) {
            const int m = it.b * kR + r;
            float mstar = NEG_INF;
#pragma unroll
            for (int w = 0; w < NCW; ++w)
                mstar = fmaxf(mstar, sm.wm[w][r]);
            float wt[NCW];
            float lstar = 0.f;
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
                const float mw = sm.wm[w][r];
                wt[w] = (mw == NEG_INF) ? 0.f : fast_exp2(mw - mstar);
                lstar = fmaf(sm.wl[w][r], wt[w], lstar);
            }
            if (m >= p.M || sm.abort_flag)
                continue;
            float *dst;
            float scale_out;
            if (it.fin) {
                const int wr = m / p.G;
                const int h = it.kh * p.G + (m - wr * p.G);
                dst = p.out + (((size_t)it.s * p.W + wr) * p.Hq + h) * D;
                scale_out = 1.f / lstar;
            } else {
                float *slot =
                    p.part + (size_t)it.slot * part_slot_floats(p);
                dst = slot + (size_t)r * D;
                scale_out = 1.f;
                if (lane == 0) {
                    slot[(size_t)p.SR * D + r] = mstar;
                    slot[(size_t)p.SR * D + p.SR + r] = lstar;
                }
            }
#pragma unroll
            for (int q4 = 0; q4 < D / 128; ++q4) {
                const int col = q4 * 128 + lane * 4;
                float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int w = 0; w < NCW; ++w) {
                    const float4 v = *reinterpret_cast<const float4 *>(&sm.wo[w][r][col]);
                    a.x = fmaf(v.x, wt[w], a.x);
                    a.y = fmaf(v.y, wt[w], a.y);
                    a.z = fmaf(v.z, wt[w], a.z);
                    a.w = fmaf(v.w, wt[w], a.w);
                }
                *reinterpret_cast<float4 *>(dst + col) =
                    make_float4(a.x * scale_out, a.y * scale_out, a.z * scale_out, a.w * scale_out);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.w_free);
    }
}

template <int D, bool kTree>
__global__ void __launch_bounds__(simt_threads<D>(), 1)
    attn_simt_kernel(const __grid_constant__ AttnParams p)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SimtSmem<D> &sm = *reinterpret_cast<SimtSmem<D> *>(smem_raw);
    allow_dependent_launch();
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < SimtSmem<D>::NSTAGE; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
            sm.stage_tile[s] = 0xffffffffu;
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.q_full[s], 1);
            mbar_init(&sm.q_empty[s], SimtCfg<D>::NCW);
        }
        mbar_init(&sm.w_free, 1);
        sm.w_count = 0;
        sm.abort_flag = 0;
        sm.wait_limit = p.wait_limit;
        fence_mbar_init();
    }
    wait_prior_grid();
    if (warp == SimtCfg<D>::NCW)
        find_range(p, sm.range, lane);
    __syncthreads();
    if (warp == SimtCfg<D>::NCW) {
        if (lane == 0)
            simt_producer<D>(p, sm);
    } else
        simt_consumer<D, kTree>(p, sm, warp, lane);
}

// Host-side launcher (same translation unit as the kernel template).
template <int D, bool kTree>
cudaError_t launch_simt(const AttnParams &p, int grid, cudaStream_t stream)
{
    const size_t smem = simt_smem_bytes<D>();
    static std::atomic<bool> configured[kMaxDevices];
    const cudaError_t e = set_smem_limit_once(attn_simt_kernel<D, kTree>, smem, configured);
    if (e != cudaSuccess)
        return e;
    return launch_dependent(attn_simt_kernel<D, kTree>, dim3(grid), dim3(simt_threads<D>()), smem,
                            stream, p);
}

template <int D>
cudaError_t launch_attn_simt(const AttnParams &p, int grid, cudaStream_t stream)
{
    return p.has_tree ? launch_simt<D, true>(p, grid, stream) : launch_simt<D, false>(p, grid, stream);
}

template cudaError_t launch_attn_simt<128>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_simt<512>(const AttnParams &, int, cudaStream_t);
template size_t simt_smem_bytes<128>();
template size_t simt_smem_bytes<512>();

}  // namespace tfp
