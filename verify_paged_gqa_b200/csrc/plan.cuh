// plan.cuh -- how one attention call is cut into work items.
//
// A unit is (stream s, KV head kh).  Its M = G * W query rows (W window
// rows times the G query heads of the group, row m = r * G + g) are cut into
// row blocks of RB rows, and the keys a row block can see are cut into
// chunks of CH positions (CH a multiple of the page size, fixed by host
// arguments only).  One work item = (s, kh, row block b, chunk c).  Items are
// numbered stream by stream, then KV head, row block, chunk; persistent CTAs
// take items round-robin.  A row block with one chunk is finished by its
// item; otherwise every item leaves a partial (unnormalised O, running max,
// running sum) in a fixed slot of the workspace and the merge kernel
// combines them in chunk order.  Which CTA runs an item never changes its
// arithmetic, so results depend only on positions, lens and host arguments.
#pragma once

#include "common.cuh"

namespace tfp {

__host__ __device__ __forceinline__ bool len_ok(const AttnParams &p, int len)
{
    return len >= p.W && len <= p.max_len && (int64_t)len <= (int64_t)p.table_stride * p.P;
}

// One past the last position any row of row block b may see.
__host__ __device__ __forceinline__ int block_lim(const AttnParams &p, int len, int b)
{
    const int m_last = min(p.M, (b + 1) * p.RB) - 1;
    return len - p.W + m_last / p.G + 1;
}

// One past the position row m sees (rows past M are clamped to the last row).
__host__ __device__ __forceinline__ int row_lim(const AttnParams &p, int len, int m)
{
    return len - p.W + min(m, p.M - 1) / p.G + 1;
}

__host__ __device__ __forceinline__ int block_chunks(const AttnParams &p, int len, int b)
{
    return (block_lim(p, len, b) + p.CH - 1) / p.CH;
}

__host__ __device__ __forceinline__ int64_t part_slot(const AttnParams &p, int s, int kh, int b,
                                                      int c)
{
    return (((int64_t)s * p.Hkv + kh) * p.n_rblk + b) * p.max_chunks + c;
}

__device__ __forceinline__ int stream_items(const AttnParams &p, int len)
{
    if (!len_ok(p, len))
        return 0;
    int n = 0;
    for (int b = 0; b < p.n_rblk; ++b)
        n += block_chunks(p, len, b);
    return n * p.Hkv;
}

struct WorkItem {
    int s, kh, b, c, nc, len;
    int key0, key1;  // positions [key0, key1) this item reads
};

// Walks the item numbering; seek() must be called with non-decreasing i.
struct ItemCursor {
    int s;
    int64_t base;
    int cnt;
    int len;

    __device__ __forceinline__ void init()
    {
        s = -1;
        base = 0;
        cnt = 0;
        len = 0;
    }

    __device__ __forceinline__ bool seek(const AttnParams &p, int64_t i, WorkItem &w)
    {
        while (i >= base + cnt) {
            base += cnt;
            ++s;
            if (s >= p.S)
                return false;
            len = __ldg(p.lens + s);
            cnt = stream_items(p, len);
        }
        const int r = static_cast<int>(i - base);
        const int per_kh = cnt / p.Hkv;
        w.s = s;
        w.len = len;
        w.kh = r / per_kh;
        int r2 = r - w.kh * per_kh;
        int b = 0;
        for (; b < p.n_rblk - 1; ++b) {
            const int nc = block_chunks(p, len, b);
            if (r2 < nc)
                break;
            r2 -= nc;
        }
        w.b = b;
        w.c = r2;
        w.nc = block_chunks(p, len, b);
        w.key0 = r2 * p.CH;
        w.key1 = min(w.key0 + p.CH, block_lim(p, len, b));
        return true;
    }
};

}  // namespace tfp
