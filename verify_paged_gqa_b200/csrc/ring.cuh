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

// ---- page sizes that are not a multiple of 128: tiles gathered row by row ----
//
// A 128-position tile may then straddle pages, and a TMA box cannot follow
// the table.  The producer warp instead copies every position's row (128
// dims of K or V: 256 bytes, 16 chunks of 16 bytes) with cp.async into the
// same 128-byte-swizzled layout the TMA boxes produce, so the MMAs read the
// ring unchanged.  Each lane arrives on the unit's full barrier once its own
// copies have landed (32 arrivals per phase).  The consumers then issue a
// proxy fence before the MMAs read the unit (cp.async writes through the
// generic proxy).

// Pool rows of the tile's positions: lane l holds position tpos + 32 i + l in
// y[i]; -1 for a position at or past the stream's end (never read: its K row
// is masked and its V row zeroed before use) or on a page outside the pool
// (never read; flagged).  Table entries past the stream's end are not read.
struct TileRows {
    int y[4];
};

__device__ __forceinline__ TileRows tile_rows(const AttnParams &p, const int32_t *trow, int kh,
                                              int tpos, int len, int lane)
{
    TileRows t;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int pos = tpos + 32 * i + lane;
        int y = -1;
        if (pos < len) {
            const int lp = pos / p.P;
            const int page = __ldg(trow + lp);
            if (page >= 0 && page < p.n_pages)
                y = (page * p.Hkv + kh) * p.P + (pos - lp * p.P);
            else
                bad = true;
        }
        t.y[i] = y;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0)
        set_flag(p.flags, kDevBadPage);
    return t;
}

// The whole warp: waits until slot st is free, then copies dims [128 kb,
// 128 kb + 128) of the tile's rows from `pool` into it.  False (uniform) when
// the wait gave up.
template <class Sm>
__device__ __forceinline__ bool gather_unit(const AttnParams &p, Sm &sm, int st, uint32_t parity,
                                            const __nv_bfloat16 *pool, const TileRows &rows,
                                            int kb, int lane, uint64_t pol)
{
    bool ok = true;
    if (lane == 0)
        ok = pwait(sm, &sm.empty[st], parity, p.flags, kWaitEmpty);
    if (!__shfl_sync(0xffffffffu, ok, 0))
        return false;
    const int ch = lane & 15;  // the lane's 16-byte chunk of a row: dims [8 ch, 8 ch + 8)
    uint8_t *const dst = sm.ring[st] + (ch >> 3) * kRingBox;
    const __nv_bfloat16 *const src = pool + kb * 128 + ch * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            // rows 32 i + 2 k (lanes 0-15) and 32 i + 2 k + 1 (lanes 16-31)
            const int j = 2 * k + (lane >> 4);
            const int y = __shfl_sync(0xffffffffu, rows.y[i], j);
            if (y >= 0)
                cp_async16(dst + sw128_off(32 * i + j, ch & 7), src + (size_t)y * p.D, pol);
        }
    }
    cp_async_arrive(&sm.full[st]);
    return true;
}

// The whole producer warp: the unit order of ring_producer, gathered.
template <int DB, int NU, class Sm>
__device__ __forceinline__ void ring_producer_gather(const AttnParams &p, Sm &sm, int lane)
{
    const uint64_t pol = l2_evict_first_policy();
    SegCursor cur;
    cur.init(p, sm.range);
    WorkItem it;
    uint32_t U = 0;  // units issued
    bool ok = true;
    auto put_tile = [&](const __nv_bfloat16 *pool, const TileRows &rows) {
#pragma unroll 1
        for (int kb = 0; ok && kb < DB; ++kb) {
            ok = gather_unit(p, sm, (int)(U % NU), ((U / NU) & 1u) ^ 1u, pool, rows, kb, lane, pol);
            U += ok ? 1u : 0u;
        }
    };
    while (ok && cur.next(p, it)) {
        const int n = (it.key1 - it.key0 + kRingTile - 1) / kRingTile;
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        TileRows r0 = tile_rows(p, trow, it.kh, it.key0, it.len, lane);
        put_tile(p.k_pool, r0);
        for (int t = 0; ok && t < n; ++t) {
            const int pos = it.key0 + t * kRingTile;
            TileRows r1 = r0;
            if (t + 1 < n) {
                r1 = tile_rows(p, trow, it.kh, pos + kRingTile, it.len, lane);
                put_tile(p.k_pool, r1);
            }
            if (ok)
                put_tile(p.v_pool, r0);
            r0 = r1;
        }
    }
    if (lane == 0) {
        // Let the copies in flight land before the CTA can exit (a unit's
        // phase completes once every lane's copies of it have landed).
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
