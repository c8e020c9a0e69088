// plan.cuh -- how one attention call is cut into work (stream-K).
//
// A unit is (stream s, KV head kh, row block b): its RB query rows (of the
// M = G * W rows of (s, kh); row m = r * G + g) and the keys they can see,
// [0, block_lim).  Those keys are cut into tiles of kTile positions.  The
// launch's units are laid end to end -- stream by stream, then KV head, then
// row block -- and their work is split evenly over the persistent CTAs.  A
// unit's work is its tiles plus VT "entry" tiles in front of them that hold
// no positions: they stand for what a CTA pays to start a unit (its query
// rows, the pipeline filling again, one more epilogue), so a CTA whose range
// crosses into a new unit gets that many fewer real tiles.  With T work
// tiles in all and G CTAs, CTA c takes [c T / G, (c + 1) T / G).  The split
// is computed on the device from the streams' actual lengths, so every CTA
// gets the same work whatever the length mix, and a captured graph stays
// valid as the lengths grow.
//
// A CTA's range meets a run of units; each meeting is a segment.  A segment
// that covers its whole unit finishes the unit's rows itself.  Otherwise it
// leaves a partial (unnormalised O, running max, running sum) in one of the
// CTA's two workspace slots: slot 2c for a segment that starts at the CTA's
// first tile, 2c + 1 for one that ends at its last (a CTA range meets at most
// two units partially).  The merge kernel finds a split unit's segments from
// the same arithmetic and combines them in position order.  (When the call's
// units fill most CTAs but not more, the tensor-bound prompt kernel instead
// gives CTA c unit c whole: no partials and no merge.)  A unit's result
// therefore depends on the lengths of the call's streams and the grid size
// (never on the page table, nor on run-to-run timing).
#pragma once

#include "common.cuh"

namespace tfp {

constexpr int kTile = 128;     // positions per scheduling tile
constexpr int kMaxCtas = 1024; // persistent CTAs of a partial kernel, at most

__host__ __device__ __forceinline__ bool len_ok(const AttnParams &p, int len)
{
    return len >= p.W && len <= p.max_len && (int64_t)len <= (int64_t)p.table_stride * p.P;
}

// One past the last position any row of row block b may see (under tree
// masks a row may see any row of its window).
__host__ __device__ __forceinline__ int block_lim(const AttnParams &p, int len, int b)
{
    if (p.has_tree)
        return len;
    const int m_last = min(p.M, (b + 1) * p.RB) - 1;
    return len - p.W + m_last / p.G + 1;
}

// One past the position row m sees (rows past M are clamped to the last row);
// causal windows only.
__host__ __device__ __forceinline__ int row_lim(const AttnParams &p, int len, int m)
{
    return len - p.W + min(m, p.M - 1) / p.G + 1;
}

__host__ __device__ __forceinline__ int unit_tiles(const AttnParams &p, int len, int b)
{
    return (block_lim(p, len, b) + kTile - 1) / kTile;
}

// Work of a unit: its entry tiles, then its tiles.
__host__ __device__ __forceinline__ int unit_work(const AttnParams &p, int len, int b)
{
    return p.VT + unit_tiles(p, len, b);
}

// Work of one KV head of a stream (all its row blocks); 0 for a length out
// of range (those streams are skipped and reported by the merge kernel).
__host__ __device__ __forceinline__ int64_t head_work(const AttnParams &p, int len)
{
    if (!len_ok(p, len))
        return 0;
    int64_t n = 0;
    for (int b = 0; b < p.n_rblk; ++b)
        n += unit_work(p, len, b);
    return n;
}

// First work tile of CTA c's range, and the CTA whose range holds work tile g.
__host__ __device__ __forceinline__ int64_t range_start(int64_t tot, int c, int n_cta)
{
    return tot * c / n_cta;
}

__host__ __device__ __forceinline__ int cta_of(int64_t g, int64_t tot, int n_cta)
{
    return static_cast<int>((g * n_cta + n_cta - 1) / tot);
}

// This CTA's range, found by warp 0 at kernel start.
struct CtaRange {
    long long g0, g1;   // work tiles [g0, g1) of the launch
    long long off0;     // g0's offset inside stream s0
    int s0;             // stream holding tile g0 (S when the range is empty)
    int pad;
};

// Run by one whole warp.  Two passes over the streams' lengths, 32 at a
// time: the total work, then the stream holding the CTA's first work tile.
// CTA 0 also records where every stream's work starts and the total in the
// workspace for the merge kernel.
__device__ __forceinline__ void find_range(const AttnParams &p, CtaRange &out, int lane)
{
    if (p.whole) {
        // CTA c takes unit c (stream, KV head, row block) whole
        const int per_s = p.Hkv * p.n_rblk;
        const int c = blockIdx.x;
        const int s = c / per_s;
        const int len = s < p.S ? __ldg(p.lens + s) : 0;
        const long long hw = s < p.S ? head_work(p, len) : 0;
        if (lane == 0) {
            out.g0 = 0;
            out.g1 = 0;
            out.off0 = 0;
            out.s0 = p.S;
            if (hw > 0) {
                const int kh = (c - s * per_s) / p.n_rblk;
                const int b = c - s * per_s - kh * p.n_rblk;
                long long before = 0;
                for (int bb = 0; bb < b; ++bb)
                    before += unit_work(p, len, bb);
                out.s0 = s;
                out.off0 = kh * hw + before;
                out.g1 = unit_work(p, len, b);
            }
        }
        return;
    }
    long long tot = 0;
    for (int s = lane; s < p.S; s += 32)
        tot += p.Hkv * head_work(p, __ldg(p.lens + s));
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1)
        tot += __shfl_xor_sync(0xffffffffu, tot, k);
    const long long g0 = range_start(tot, blockIdx.x, gridDim.x);
    const long long g1 = range_start(tot, blockIdx.x + 1, gridDim.x);
    const bool writer = blockIdx.x == 0;
    int s0 = p.S;
    long long off0 = 0, base = 0;
    for (int c0 = 0; c0 < p.S && (writer || (g0 < g1 && s0 == p.S)); c0 += 32) {
        const int s = c0 + lane;
        const long long t = s < p.S ? p.Hkv * head_work(p, __ldg(p.lens + s)) : 0;
        long long incl = t;
#pragma unroll
        for (int k = 1; k < 32; k <<= 1) {
            const long long v = __shfl_up_sync(0xffffffffu, incl, k);
            if (lane >= k)
                incl += v;
        }
        const long long excl = base + incl - t;
        if (writer && s < p.S)
            p.first_tile[s] = excl;
        const unsigned hit = __ballot_sync(0xffffffffu, t > 0 && excl <= g0 && g0 < excl + t);
        if (hit != 0 && s0 == p.S) {
            const int L = __ffs(hit) - 1;
            s0 = c0 + L;
            off0 = g0 - __shfl_sync(0xffffffffu, excl, L);
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (writer && lane == 0)
        *p.total_tiles = tot;
    if (lane == 0) {
        out.g0 = g0;
        out.g1 = g1;
        out.off0 = off0;
        out.s0 = g0 < g1 ? s0 : p.S;
    }
}

struct WorkItem {
    int s, kh, b, len;
    int key0, key1;  // positions [key0, key1) this segment reads
    bool fin;        // covers the whole unit: write the rows' outputs
    int slot;        // partial slot otherwise
};

// Walks this CTA's segments in order; each role of a CTA keeps its own.  A
// part of the range that holds only a unit's entry tiles yields no segment.
struct SegCursor {
    int s, kh, b, off, len;   // off: work tiles of unit (s, kh, b) already passed
    long long left;
    bool first;

    __device__ __forceinline__ void init(const AttnParams &p, const CtaRange &r)
    {
        left = r.g1 - r.g0;
        first = true;
        s = r.s0;
        kh = b = off = 0;
        len = 0;
        if (left <= 0 || s >= p.S) {
            left = 0;
            return;
        }
        len = __ldg(p.lens + s);
        const long long hw = head_work(p, len);
        kh = static_cast<int>(r.off0 / hw);
        int rem = static_cast<int>(r.off0 - kh * hw);
        for (;;) {
            const int wu = unit_work(p, len, b);
            if (rem < wu)
                break;
            rem -= wu;
            ++b;
        }
        off = rem;
    }

    __device__ __forceinline__ bool next(const AttnParams &p, WorkItem &w)
    {
        while (left > 0) {
            const int wu = unit_work(p, len, b);
            const int n = static_cast<int>(min((long long)(wu - off), left));
            const int t0 = max(off - p.VT, 0), t1 = max(off + n - p.VT, 0);  // real tiles
            const bool emit = t1 > t0;
            if (emit) {
                w.s = s;
                w.kh = kh;
                w.b = b;
                w.len = len;
                w.key0 = t0 * kTile;
                w.key1 = min(t1 * kTile, block_lim(p, len, b));
                w.fin = t0 == 0 && t1 == wu - p.VT;
                w.slot = w.fin ? -1 : 2 * static_cast<int>(blockIdx.x) + (first ? 0 : 1);
                first = false;
            }
            left -= n;
            off += n;
            if (left > 0) {
                // the next unit with work
                off = 0;
                if (++b == p.n_rblk) {
                    b = 0;
                    if (++kh == p.Hkv) {
                        kh = 0;
                        do {
                            ++s;
                            len = s < p.S ? __ldg(p.lens + s) : 0;
                        } while (s < p.S && head_work(p, len) == 0);
                        if (s >= p.S)
                            left = 0;
                    }
                }
            }
            if (emit)
                return true;
        }
        return false;
    }
};

}  // namespace tfp
