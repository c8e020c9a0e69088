// ring.cuh -- the K/V ring shared by the two tensor-core partial kernels.
//
// A ring unit is 128 key positions x 128 head dims of one page x KV head
// (K or V), loaded by TMA as two [128][64] bf16 boxes with 128-byte swizzle.
// A tile of 128 positions at head dim D is DB = D / 128 units of K and DB of
// V.  The producer loads, per segment, K(0) and then for each tile t the K
// units of tile t + 1 (if any) followed by the V units of tile t: the MMA
// issuer runs QK(t + 1) before PV(t), so it consumes the units in exactly
// this order.  The kernel's shared-memory struct provides ring[NU][kRingUnit],
// full[NU], empty[NU], range and abort_flag.
#pragma once

#include "plan.cuh"
#include "umma.cuh"

namespace tfp {

constexpr int kRingTile = 128;             // positions per tile
constexpr uint32_t kRingBox = 16384;       // one [128 positions][64 dims] bf16 box
constexpr uint32_t kRingUnit = 2 * kRingBox;

// mbarrier wait that records a timeout (status bit and wait site) and makes
// every role of the CTA wind down.
template <class Sm>
__device__ __forceinline__ bool pwait(Sm &sm, uint64_t *bar, uint32_t parity, uint32_t *flags,
                                      uint32_t site)
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

// OR of `pred` over the NT threads of named barrier 1.
template <int NT>
__device__ __forceinline__ bool block_any(bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, %2, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(NT)
        : "memory");
    return r != 0;
}

// Loads the DB units of one K or V tile (positions [off, off + 128) of a page).
template <int DB, int NU, class Sm>
__device__ __forceinline__ bool ring_put_tile(const AttnParams &p, Sm &sm, uint32_t &U,
                                              const CUtensorMap *map, int page, int kh, int off,
                                              uint64_t pol)
{
    const bool page_ok = page >= 0 && page < p.n_pages;
    if (!page_ok)
        set_flag(p.flags, kDevBadPage);
    const int y = ((page_ok ? page : 0) * p.Hkv + kh) * p.P + off;
#pragma unroll 1
    for (int kb = 0; kb < DB; ++kb) {
        const int st = (int)(U % NU);
        if (!pwait(sm, &sm.empty[st], ((U / NU) & 1u) ^ 1u, p.flags, kWaitEmpty))
            return false;
        if (page_ok) {
            mbar_arrive_expect_tx(&sm.full[st], kRingUnit);
            tma_load_2d(sm.ring[st], map, 128 * kb, y, &sm.full[st], pol);
            tma_load_2d(sm.ring[st] + kRingBox, map, 128 * kb + 64, y, &sm.full[st], pol);
        } else {
            mbar_arrive(&sm.full[st]);
        }
        ++U;
    }
    return true;
}

// One lane runs this.  Page ids are read two tiles ahead.
template <int DB, int NU, class Sm>
__device__ __forceinline__ void ring_producer(const AttnParams &p, const CUtensorMap *kmap,
                                              const CUtensorMap *vmap, Sm &sm)
{
    constexpr int PT = kRingTile;
    const uint64_t pol = l2_evict_first_policy();
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t U = 0;
    bool ok = true;
    while (ok && cur.next(p, it)) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        int pg0 = __ldg(trow + it.key0 / p.P);
        int pg1 = n > 1 ? __ldg(trow + (it.key0 + PT) / p.P) : 0;
        ok = ring_put_tile<DB, NU>(p, sm, U, kmap, pg0, it.kh, it.key0 % p.P, pol);
        for (int t = 0; ok && t < n; ++t) {
            const int pos = it.key0 + t * PT;
            const int pg2 = t + 2 < n ? __ldg(trow + (pos + 2 * PT) / p.P) : 0;
            if (t + 1 < n)
                ok = ring_put_tile<DB, NU>(p, sm, U, kmap, pg1, it.kh, (pos + PT) % p.P, pol);
            if (ok)
                ok = ring_put_tile<DB, NU>(p, sm, U, vmap, pg0, it.kh, pos % p.P, pol);
            pg0 = pg1;
            pg1 = pg2;
        }
    }
    {
        // Let the copies in flight land before the CTA can exit.  On the
        // normal path every unit was consumed and these phases are complete;
        // after another role gave up, some may still be in flight.
        const uint32_t nf = U < (uint32_t)NU ? U : (uint32_t)NU;
        for (uint32_t k = 1; k <= nf; ++k) {
            const uint32_t v = U - k;
            (void)mbar_wait(&sm.full[v % NU], (v / NU) & 1u, p.wait_limit);
        }
    }
}

// ---- page sizes that are not a multiple of 128: tiles assembled from pages ----
//
// A 128-position tile may then straddle pages, and one box of 128 rows cannot
// follow the table.  The tile is cut into pieces, one per page it touches,
// and each piece of n rows is loaded with one 2-D TMA box per set bit of n
// (box heights 1, 2, 4, ..., 128 rows, one tensor map each), each landing at
// its own tile row.  The 128-byte swizzle is a function of the shared-memory
// address, so the pieces form the same layout a single 128-row box gives and
// the MMAs read the ring unchanged.  Rows at or past the stream's end are not
// loaded (their K rows are masked and their V rows zeroed before use), and
// the unit completes on its full barrier by bytes.

constexpr int kBoxHeights = 8;  // tensor maps of boxes 1, 2, 4, ..., 128 rows high

// The pages of a tile's valid rows [tpos, tpos + nvalid): the first is page
// lp0, entered at slot off0; lane l holds the id of page lp0 + l (the first 32
// pages the rows touch).  Table entries past the stream's pages are not read.
struct TilePages {
    int lp0, off0;
    int id;
};

__device__ __forceinline__ TilePages tile_pages(const AttnParams &p, const int32_t *trow, int tpos,
                                                int nvalid, int lane)
{
    TilePages t;
    t.lp0 = tpos / p.P;
    t.off0 = tpos - t.lp0 * p.P;
    // page lp0 + lane starts at tile row lane * P - off0: does it hold a valid row?
    const bool mine = (int64_t)lane * p.P < (int64_t)t.off0 + nvalid;
    t.id = mine ? __ldg(trow + t.lp0 + lane) : 0;
    return t;
}

// The whole warp (lane 0 issues): waits until slot st is free, then loads
// dims [128 kb, 128 kb + 128) of the tile's valid rows through `maps` (the K
// or V pool, box heights 2^h) into it.  False (uniform) when the wait gave up.
template <class Sm>
__device__ __forceinline__ bool pieces_unit(const AttnParams &p, Sm &sm, int st, uint32_t parity,
                                            const CUtensorMap *maps, const TilePages &tp,
                                            const int32_t *trow, int kh, int nvalid, int kb,
                                            int lane, uint64_t pol)
{
    bool ok = true;
    if (lane == 0) {
        ok = pwait(sm, &sm.empty[st], parity, p.flags, kWaitEmpty);
        if (ok)
            mbar_arrive_expect_tx(&sm.full[st], (uint32_t)nvalid * 256u);
    }
    if (!__shfl_sync(0xffffffffu, ok, 0))
        return false;
    // one piece per page: rows [r, r + n) of the tile from page lp0 + j,
    // slots [off, off + n)
    int off = tp.off0;
    for (int r = 0, j = 0; r < nvalid; ++j) {
        const int n = min(nvalid - r, p.P - off);
        int page = j < 32 ? __shfl_sync(0xffffffffu, tp.id, j) : __ldg(trow + tp.lp0 + j);
        if (lane == 0) {
            if (page < 0 || page >= p.n_pages) {
                // never read: page 0 stands in (the stream's outputs are flagged)
                set_flag(p.flags, kDevBadPage);
                page = 0;
            }
            int row = r, y = (page * p.Hkv + kh) * p.P + off;
            for (int m = n; m != 0;) {
                const int h = 31 - __clz(m);  // the largest box that fits: 2^h rows
                tma_load_2d(sm.ring[st] + row * 128, &maps[h], 128 * kb, y, &sm.full[st], pol);
                tma_load_2d(sm.ring[st] + kRingBox + row * 128, &maps[h], 128 * kb + 64, y,
                            &sm.full[st], pol);
                row += 1 << h;
                y += 1 << h;
                m -= 1 << h;
            }
        }
        r += n;
        off = 0;
    }
    return true;
}

// The whole producer warp: the unit order of ring_producer, assembled from
// pieces.  kmaps / vmaps: kBoxHeights tensor maps each.
template <int DB, int NU, class Sm>
__device__ __forceinline__ void ring_producer_pieces(const AttnParams &p, const CUtensorMap *kmaps,
                                                     const CUtensorMap *vmaps, Sm &sm, int lane)
{
    const uint64_t pol = l2_evict_first_policy();
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t U = 0;  // units issued
    bool ok = true;
    auto put_tile = [&](const CUtensorMap *maps, const TilePages &tp, const int32_t *trow, int kh,
                        int nvalid) {
#pragma unroll 1
        for (int kb = 0; ok && kb < DB; ++kb) {
            ok = pieces_unit(p, sm, (int)(U % NU), ((U / NU) & 1u) ^ 1u, maps, tp, trow, kh, nvalid,
                             kb, lane, pol);
            U += ok ? 1u : 0u;
        }
    };
    constexpr int PT = kRingTile;
    while (ok && cur.next(p, it)) {
        const int n = (it.key1 - it.key0 + PT - 1) / PT;
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        // rows and page ids of tiles t, t + 1 and t + 2 (the page ids are read
        // two tiles before their first use)
        auto nvalid = [&](int t) { return min(PT, it.len - (it.key0 + t * PT)); };
        TilePages t0 = tile_pages(p, trow, it.key0, nvalid(0), lane);
        TilePages t1 = n > 1 ? tile_pages(p, trow, it.key0 + PT, nvalid(1), lane) : t0;
        put_tile(kmaps, t0, trow, it.kh, nvalid(0));
        for (int t = 0; ok && t < n; ++t) {
            const int pos = it.key0 + t * PT;
            const TilePages t2 = t + 2 < n ? tile_pages(p, trow, pos + 2 * PT, nvalid(t + 2), lane) : t1;
            if (t + 1 < n)
                put_tile(kmaps, t1, trow, it.kh, nvalid(t + 1));
            if (ok)
                put_tile(vmaps, t0, trow, it.kh, nvalid(t));
            t0 = t1;
            t1 = t2;
        }
    }
    if (lane == 0) {
        // let the copies in flight land before the CTA can exit
        const uint32_t nf = U < (uint32_t)NU ? U : (uint32_t)NU;
        for (uint32_t k = 1; k <= nf; ++k) {
            const uint32_t v = U - k;
            (void)mbar_wait(&sm.full[v % NU], (v / NU) & 1u, p.wait_limit);
        }
    }
    __syncwarp();
}

// Ring index of the first V unit of tile t of a segment that starts at the
// CTA's tile u0 and has n tiles (the order above).
__device__ __forceinline__ uint32_t ring_v_unit(int DB, uint32_t u0, int t, int n)
{
    return 2u * DB * u0 + DB * (2u * t + 1u + (t + 1 < n ? 1u : 0u));
}

}  // namespace tfp
