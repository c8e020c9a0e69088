// attn_merge.cu -- combines the split-context partials of each row block.
//
// TensorFold #1620, the comment on per-tile lookup and the reply on the
// merge: decode is split across the context by a partial kernel and put back
// together by a merge kernel that reads no pages.  For a row with partials
// (O_c, m_c, l_c), c = 0..nc-1 (O_c unnormalised, m_c the running max in log2
// units, l_c the running sum relative to m_c):
//     m* = max_c m_c,   w_c = 2^(m_c - m*),
//     out = (sum_c w_c O_c) / (sum_c w_c l_c)
// The maximum and the sum of l are warp-shuffle reductions; the O sum runs
// in segment (position) order, so the result is the same on every run.
//
// The segments of a unit split across CTAs are found from the work split
// (plan.cuh): the CTAs whose ranges meet the unit's real tiles, in order.
// One block per (stream, KV head, row block, group of up to 8 rows); one
// warp per row.  A row's first round of O loads and its (m, l) loads are all
// in flight together.  The kernel is launched as a programmatic dependent of
// the partial kernel, so its launch overlaps that kernel's last CTAs.
// Streams whose length is out of range get NaN rows (and the status bit).
#include "launch.cuh"
#include "plan.cuh"

namespace tfp {

constexpr int kMergeRows = 8;    // rows (warps) per merge block

template <int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(const __grid_constant__ AttnParams p)
{
    constexpr int DL = D / 32;            // output floats per lane
    constexpr int NV = DL / 4;            // float4 per lane and segment
    constexpr int UK = D == 128 ? 8 : 4;  // segments loaded per round
    __shared__ int slots[kMaxCtas];       // partial slot of each segment, -1: none
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int nwarps = blockDim.x / 32;
    const int groups = (p.RB + kMergeRows - 1) / kMergeRows;
    const int blk = blockIdx.x;
    const int g = blk % groups;
    const int b = (blk / groups) % p.n_rblk;
    const int u = blk / groups / p.n_rblk;
    const int kh = u % p.Hkv;
    const int s = u / p.Hkv;
    const int len = __ldg(p.lens + s);
    const int mb = b * p.RB;                       // first row of the row block
    const int m0 = mb + g * kMergeRows;
    const int m1 = min(min(p.M, mb + p.RB), m0 + kMergeRows);
    if (m0 >= m1)
        return;
    const float NEG_INF = -__int_as_float(0x7f800000);
    // launched as a programmatic dependent of the partial kernel: wait for
    // that grid to complete (and its writes to be visible) before going on
    wait_prior_grid();

    if (!len_ok(p, len)) {
        if (threadIdx.x == 0 && kh == 0 && b == 0 && g == 0)
            set_flag(p.flags, kDevBadLen);
        const float nan = __int_as_float(0x7fc00000);
        for (int m = m0 + warp; m < m1; m += nwarps) {
            const int wr = m / p.G;
            const int h = kh * p.G + (m - wr * p.G);
            float *orow = p.out + (((size_t)s * p.W + wr) * p.Hq + h) * D;
            for (int e = lane * 4; e < D; e += 128)
                *reinterpret_cast<float4 *>(orow + e) = make_float4(nan, nan, nan, nan);
        }
        return;
    }
    if (p.whole)
        return;  // every unit was finished whole by one CTA
    // the unit's tiles [U0, U1) and the CTAs that met them: warp 0 works them
    // out once for the block (lanes split the row blocks)
    __shared__ int nseg_sh;
    if (warp == 0) {
        long long hw = 0, before = 0;
        for (int bb = lane; bb < p.n_rblk; bb += 32) {
            const int t = unit_work(p, len, bb);
            hw += t;
            if (bb < b)
                before += t;
        }
#pragma unroll
        for (int k = 16; k >= 1; k >>= 1) {
            hw += __shfl_xor_sync(0xffffffffu, hw, k);
            before += __shfl_xor_sync(0xffffffffu, before, k);
        }
        const long long tot = *p.total_tiles;
        // the unit's work [U0, U1): entry tiles, then its tiles from U0 + VT
        const long long U0 = p.first_tile[s] + kh * hw + before;
        const long long U1 = U0 + unit_work(p, len, b);
        const int c_lo = cta_of(U0 + p.VT, tot, p.n_cta);
        const int c_hi = cta_of(U1 - 1, tot, p.n_cta);
        const int n = min(c_hi - c_lo + 1, kMaxCtas);
        for (int k = lane; k < n; k += 32) {
            const int c = c_lo + k;
            const long long a0 = range_start(tot, c, p.n_cta);
            const long long a1 = range_start(tot, c + 1, p.n_cta);
            // the first CTA's segment is its last unless its range starts at U0
            slots[k] = a0 == a1 ? -1 : (k == 0 && a0 < U0) ? 2 * c + 1 : 2 * c;
        }
        // one segment covered the unit and wrote the rows itself
        if (lane == 0)
            nseg_sh = c_lo == c_hi ? 0 : n;
    }
    __syncthreads();
    const int nseg = nseg_sh;
    if (nseg == 0)
        return;
    const size_t slot_floats = part_slot_floats(p);

    for (int m = m0 + warp; m < m1; m += nwarps) {
        const int r = m - mb;
        // The first round's O rows and the (m, l) of segments 0 .. 31 are
        // loaded before any of them is used, so that one memory round trip
        // covers a row with up to UK segments.
        float w[UK];
        float4 v[UK][NV];
#pragma unroll
        for (int kk = 0; kk < UK; ++kk) {
            const int sl = kk < nseg ? slots[kk] : -1;
#pragma unroll
            for (int q = 0; q < NV; ++q)
                v[kk][q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (sl >= 0) {
                const float *base = p.part + sl * slot_floats;
#pragma unroll
                for (int q = 0; q < NV; ++q)
                    v[kk][q] = *reinterpret_cast<const float4 *>(base + (size_t)r * D + q * 128 +
                                                                 lane * 4);
            }
        }
        float m_lane = NEG_INF, l_lane = 0.f;  // segment k = lane
        {
            const int sl = lane < nseg ? slots[lane] : -1;
            if (sl >= 0) {
                m_lane = p.part[sl * slot_floats + (size_t)p.SR * D + r];
                l_lane = p.part[sl * slot_floats + (size_t)p.SR * D + p.SR + r];
            }
        }
        float mx = m_lane;
        for (int k = lane + 32; k < nseg; k += 32) {
            const int sl = slots[k];
            if (sl >= 0)
                mx = fmaxf(mx, p.part[sl * slot_floats + (size_t)p.SR * D + r]);
        }
#pragma unroll
        for (int k = 16; k >= 1; k >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, k));
        float l = (m_lane == NEG_INF) ? 0.f : l_lane * fast_exp2(m_lane - mx);
        for (int k = lane + 32; k < nseg; k += 32) {
            const int sl = slots[k];
            if (sl < 0)
                continue;
            const float mc = p.part[sl * slot_floats + (size_t)p.SR * D + r];
            const float lc = p.part[sl * slot_floats + (size_t)p.SR * D + p.SR + r];
            l += (mc == NEG_INF) ? 0.f : lc * fast_exp2(mc - mx);
        }
#pragma unroll
        for (int k = 16; k >= 1; k >>= 1)
            l += __shfl_xor_sync(0xffffffffu, l, k);

        float acc[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e)
            acc[e] = 0.f;
        for (int k0 = 0; k0 < nseg; k0 += UK) {
            if (k0 > 0) {
#pragma unroll
                for (int kk = 0; kk < UK; ++kk) {
                    const int sl = k0 + kk < nseg ? slots[k0 + kk] : -1;
#pragma unroll
                    for (int q = 0; q < NV; ++q)
                        v[kk][q] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (sl >= 0) {
                        const float *base = p.part + sl * slot_floats;
#pragma unroll
                        for (int q = 0; q < NV; ++q)
                            v[kk][q] = *reinterpret_cast<const float4 *>(
                                base + (size_t)r * D + q * 128 + lane * 4);
                    }
                }
            }
            // the weights, from the (m, l) loads above where the segment has a lane
#pragma unroll
            for (int kk = 0; kk < UK; ++kk) {
                const int k = k0 + kk;
                const int sl = k < nseg ? slots[k] : -1;
                float mc = __shfl_sync(0xffffffffu, m_lane, k & 31);
                if (k >= 32 && sl >= 0)
                    mc = p.part[sl * slot_floats + (size_t)p.SR * D + r];
                w[kk] = (sl < 0 || mc == NEG_INF) ? 0.f : fast_exp2(mc - mx);
            }
#pragma unroll
            for (int kk = 0; kk < UK; ++kk) {
#pragma unroll
                for (int q = 0; q < NV; ++q) {
                    acc[q * 4 + 0] = fmaf(w[kk], v[kk][q].x, acc[q * 4 + 0]);
                    acc[q * 4 + 1] = fmaf(w[kk], v[kk][q].y, acc[q * 4 + 1]);
                    acc[q * 4 + 2] = fmaf(w[kk], v[kk][q].z, acc[q * 4 + 2]);
                    acc[q * 4 + 3] = fmaf(w[kk], v[kk][q].w, acc[q * 4 + 3]);
                }
            }
        }
        const float inv = 1.f / l;
        const int wr = m / p.G;
        const int h = kh * p.G + (m - wr * p.G);
        float *orow = p.out + (((size_t)s * p.W + wr) * p.Hq + h) * D;
#pragma unroll
        for (int q = 0; q < NV; ++q)
            *reinterpret_cast<float4 *>(orow + q * 128 + lane * 4) =
                make_float4(acc[q * 4 + 0] * inv, acc[q * 4 + 1] * inv, acc[q * 4 + 2] * inv,
                            acc[q * 4 + 3] * inv);
    }
}

template <int D>
cudaError_t launch_attn_merge(const AttnParams &p, cudaStream_t stream)
{
    const int groups = (p.RB + kMergeRows - 1) / kMergeRows;
    const int64_t blocks = (int64_t)p.S * p.Hkv * p.n_rblk * groups;
    if (blocks == 0)
        return cudaSuccess;
    const int threads = 32 * min(kMergeRows, p.RB);
    // programmatic dependent launch: the blocks are scheduled while the
    // partial kernel runs out and wait for it in the kernel
    return launch_dependent(attn_merge_kernel<D>, dim3(static_cast<unsigned>(blocks)), dim3(threads),
                            0, stream, p);
}

template cudaError_t launch_attn_merge<128>(const AttnParams &, cudaStream_t);
template cudaError_t launch_attn_merge<256>(const AttnParams &, cudaStream_t);
template cudaError_t launch_attn_merge<512>(const AttnParams &, cudaStream_t);

}  // namespace tfp
