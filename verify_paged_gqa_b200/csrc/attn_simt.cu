// attn_simt.cu -- split-context paged attention on CUDA cores, for row
// blocks of four query rows (single-row decode at GQA 4, and any small
// row count).
//
// TensorFold #1620 ("Kolibri-1's full layers take their K/V from pages of
// the core pool"): decode reads keys through the page table, split across
// the context (the partial kernel) and merged (the merge kernel, which reads
// no pages); its later comment moves the page lookup out of the per-key loop
// to once per tile.  Here one lookup serves a whole page.
//
// Layout of one CTA (persistent, one per SM):
//   last warp     producer: walks the CTA's work items, looks each page up
//                 once, and streams K and V tiles of TK positions into a ring
//                 of NSTAGE shared-memory stages with bulk copies (TMA engine,
//                 no tensor map: a tile of a page-head is one contiguous run).
//   other warps   consumers (8 at head dim 128): tile T of the CTA's
//                 sequence goes to consumer warp T % (number of consumers).
//                 A warp keeps its own online-softmax state (running max m,
//                 running sum l, unnormalised O) for the four rows of the
//                 item; at the end of the item the warps' states are combined
//                 through shared memory and the item's result is written:
//                 the normalised output when the row block has one chunk,
//                 else a partial for the merge kernel.
//
// Inner loop of a consumer warp on one tile (head dim 128, TK = 32):
//   scores  the warp is 4 groups of 8 lanes; group g takes 8 keys, lane i of
//           a group holds 16 of the 128 dims of the 4 query rows (fp32 in
//           registers) and accumulates 8 keys x 4 rows partial dots; three
//           butterfly rounds (reduce-scatter over the 8 lanes) leave lane L
//           with the 4 rows' full scores of key L.
//   softmax tile max per row by warp shuffles, exp2 of log2-scaled scores;
//           masked positions are SELECTED to -inf (never multiplied), so NaN
//           in unused slots cannot leak.
//   PV      lane L owns dims 4L..4L+3 of the 4 output rows; probabilities
//           come from a small per-warp shared buffer; only positions below
//           the item's end are visited, so no unused slot is ever read.
// Head dim 512 uses TK = 8 and one group of 32 lanes; the same steps.
#include "launch.cuh"
#include "plan.cuh"

namespace tfp {

template <int D>
struct SimtCfg;
// Registers are split per SM sub-partition: with 9 warps one sub-partition
// holds 3 warps (at most 168 registers each), with 8 warps 2 (255 each).
// Head dim 512 keeps 64 output accumulators per lane and takes 7 consumers.
template <>
struct SimtCfg<128> {
    static constexpr int TK = 32;      // positions per tile
    static constexpr int LG = 8;       // lanes sharing one key's dot product
    static constexpr int NSTAGE = 12;  // ring depth (16 KB per stage)
    static constexpr int NCW = 8;      // consumer warps
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
    static constexpr int TILE_BYTES = TK * D * 2;
    alignas(128) uint8_t kv[NSTAGE][2][TILE_BYTES];
    static constexpr int NCW = SimtCfg<D>::NCW;
    alignas(16) float pbuf[NCW][TK * kR];
    alignas(16) float wo[NCW][kR][D];
    float wm[NCW][kR];
    float wl[NCW][kR];
    uint64_t full[NSTAGE];
    uint64_t empty[NSTAGE];
    volatile int abort_flag;
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

template <int D>
__device__ __forceinline__ void simt_producer(const AttnParams &p, SimtSmem<D> &sm)
{
    constexpr int TK = SimtCfg<D>::TK;
    constexpr int NSTAGE = SimtCfg<D>::NSTAGE;
    const uint64_t pol = l2_evict_first_policy();
    ItemCursor cur;
    cur.init();
    WorkItem it;
    uint32_t T = 0;
    bool aborted = false;
    for (int64_t i = blockIdx.x; !aborted && cur.seek(p, i, it); i += gridDim.x) {
        const int32_t *trow = p.table + (int64_t)it.s * p.table_stride;
        int lp_cached = -1;
        int32_t page = 0;
        for (int t0 = it.key0; t0 < it.key1; t0 += TK, ++T) {
            const int stage = T % NSTAGE;
            const uint32_t ph = (T / NSTAGE) & 1u;
            if (!mbar_wait(&sm.empty[stage], ph ^ 1u)) {
                set_flag(p.flags, kDevTimeout);
                sm.abort_flag = 1;
                aborted = true;
                break;
            }
            const int lp = t0 / p.P;
            if (lp != lp_cached) {  // one table read per page
                page = __ldg(trow + lp);
                lp_cached = lp;
            }
            const int nk = min(TK, it.key1 - t0);
            const uint32_t bytes = static_cast<uint32_t>(nk) * D * 2u;
            if (page >= 0 && page < p.n_pages) {
                const size_t off = (((size_t)page * p.Hkv + it.kh) * p.P + (t0 - lp * p.P)) * D;
                mbar_arrive_expect_tx(&sm.full[stage], 2u * bytes);
                bulk_g2s(sm.kv[stage][0], p.k_pool + off, bytes, &sm.full[stage], pol);
                bulk_g2s(sm.kv[stage][1], p.v_pool + off, bytes, &sm.full[stage], pol);
            } else {
                set_flag(p.flags, kDevBadPage);
                mbar_arrive(&sm.full[stage]);
            }
        }
    }
    if (aborted) {
        // Let every copy this CTA started land before the CTA can exit.
        const uint32_t n = T < (uint32_t)NSTAGE ? T : (uint32_t)NSTAGE;
        for (uint32_t k = 1; k <= n; ++k) {
            const uint32_t t = T - k;
            (void)mbar_wait(&sm.full[t % NSTAGE], (t / NSTAGE) & 1u);
        }
    }
}

template <int D>
__device__ __forceinline__ void simt_consumer(const AttnParams &p, SimtSmem<D> &sm, int warp,
                                              int lane)
{
    constexpr int TK = SimtCfg<D>::TK;
    constexpr int NSTAGE = SimtCfg<D>::NSTAGE;
    constexpr int LG = SimtCfg<D>::LG;
    constexpr int NG = 32 / LG;        // key groups per warp
    constexpr int KPG = TK / NG;       // keys per group
    constexpr int NACC = KPG * kR;     // partial dots per lane
    constexpr int NV = NACC / LG;      // full scores per lane after the reduce-scatter
    constexpr int CPL = D / 8 / LG;    // 16-byte chunks of a key row per lane
    constexpr int DL = D / 32;         // output dims per lane
    constexpr int kNCW = SimtCfg<D>::NCW;
    static_assert(NACC == 32 && CPL == 2, "tile shape");
    static_assert(NV == kR || NV == 1, "score ownership");

    const int grp = lane / LG;
    const int li = lane % LG;
    const float NEG_INF = -__int_as_float(0x7f800000);

    ItemCursor cur;
    cur.init();
    WorkItem it;
    uint32_t T0 = 0;  // CTA tile index of the item's first tile

    for (int64_t i = blockIdx.x; cur.seek(p, i, it); i += gridDim.x) {
        // --- this item's query rows, fp32 in registers --------------------
        float qv[kR][CPL * 8];
        int lim[kR];
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            const int m = it.b * kR + r;
            const int mm = min(m, p.M - 1);
            const int wr = mm / p.G;
            const int h = it.kh * p.G + (mm - wr * p.G);
            lim[r] = row_lim(p, it.len, m);
            const __nv_bfloat16 *qrow = p.q + (((size_t)it.s * p.W + wr) * p.Hq + h) * D;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const uint4 w = *reinterpret_cast<const uint4 *>(qrow + (li + c * LG) * 8);
                const bool live = m < p.M;
                qv[r][c * 8 + 0] = live ? bf_lo(w.x) : 0.f;
                qv[r][c * 8 + 1] = live ? bf_hi(w.x) : 0.f;
                qv[r][c * 8 + 2] = live ? bf_lo(w.y) : 0.f;
                qv[r][c * 8 + 3] = live ? bf_hi(w.y) : 0.f;
                qv[r][c * 8 + 4] = live ? bf_lo(w.z) : 0.f;
                qv[r][c * 8 + 5] = live ? bf_hi(w.z) : 0.f;
                qv[r][c * 8 + 6] = live ? bf_lo(w.w) : 0.f;
                qv[r][c * 8 + 7] = live ? bf_hi(w.w) : 0.f;
            }
        }

        float m_run[kR], l_lane[NV], o[kR][DL];
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            m_run[r] = NEG_INF;
#pragma unroll
            for (int e = 0; e < DL; ++e)
                o[r][e] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < NV; ++j)
            l_lane[j] = 0.f;

        const int ntiles = (it.key1 - it.key0 + TK - 1) / TK;
        int t = (warp - (int)(T0 % kNCW) + kNCW) % kNCW;
        for (; t < ntiles; t += kNCW) {
            const uint32_t T = T0 + t;
            const int stage = T % NSTAGE;
            if (!sm.abort_flag && !mbar_wait(&sm.full[stage], (T / NSTAGE) & 1u)) {
                if (lane == 0)
                    set_flag(p.flags, kDevTimeout);
                sm.abort_flag = 1;
            }
            __syncwarp();
            if (sm.abort_flag)
                continue;
            const uint8_t *Ks = sm.kv[stage][0];
            const uint8_t *Vs = sm.kv[stage][1];
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
                    const float kf[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                                         bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
                    for (int r = 0; r < kR; ++r) {
                        float a = acc[kk * kR + r];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            a = fmaf(qv[r][c * 8 + e], kf[e], a);
                        acc[kk * kR + r] = a;
                    }
                }
            }
            // --- reduce-scatter over the LG lanes of the group -------------
            // Round with mask msk keeps the upper half of the array in lanes
            // whose bit msk is set.  Afterwards lane li holds entries
            // x = li * NV + j (j < NV) of the original kk * kR + r numbering.
            constexpr int LOG_LG = (LG == 8) ? 3 : 5;
            static_assert((1 << LOG_LG) == LG, "lane group");
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
                    const bool vis = key < nk && pos < lim[r];
                    sc[r] = vis ? acc[r] * p.scale_log2 : NEG_INF;
                    tmax[r] = warp_max(sc[r], 1);
                }
            } else {
                const int key = li >> 2;
                const int r = li & 3;
                const int pos = tpos + key;
                const int my_lim = r == 0 ? lim[0] : r == 1 ? lim[1] : r == 2 ? lim[2] : lim[3];
                const bool vis = key < nk && pos < my_lim;
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
            float *pb = sm.pbuf[warp];
            if constexpr (NV == kR) {
                float pr[kR];
#pragma unroll
                for (int r = 0; r < kR; ++r) {
                    pr[r] = fast_exp2(sc[r] - m_use[r]);
                    l_lane[r] = fmaf(l_lane[r], alpha[r], pr[r]);
                }
                *reinterpret_cast<float4 *>(pb + lane * 4) = make_float4(pr[0], pr[1], pr[2], pr[3]);
            } else {
                const int r = li & 3;
                const float mu = r == 0 ? m_use[0] : r == 1 ? m_use[1] : r == 2 ? m_use[2] : m_use[3];
                const float al = r == 0 ? alpha[0] : r == 1 ? alpha[1] : r == 2 ? alpha[2] : alpha[3];
                const float pr = fast_exp2(sc[0] - mu);
                l_lane[0] = fmaf(l_lane[0], al, pr);
                pb[lane] = pr;
            }
            __syncwarp();

            // --- O = alpha * O + P V over the visited positions -----------
#pragma unroll
            for (int r = 0; r < kR; ++r)
#pragma unroll
                for (int e = 0; e < DL; ++e)
                    o[r][e] *= alpha[r];

            auto pv_step = [&](int kk) {
                const float4 pr = *reinterpret_cast<const float4 *>(pb + kk * 4);
                const float prr[4] = {pr.x, pr.y, pr.z, pr.w};
                if constexpr (D == 128) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(Vs + kk * D * 2 + lane * 8);
                    const float v[4] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y)};
#pragma unroll
                    for (int r = 0; r < kR; ++r)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            o[r][e] = fmaf(prr[r], v[e], o[r][e]);
                } else {
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(Vs + kk * D * 2 + lane * 16);
                    const uint4 w1 =
                        *reinterpret_cast<const uint4 *>(Vs + kk * D * 2 + D + lane * 16);
                    const float v[16] = {bf_lo(w0.x), bf_hi(w0.x), bf_lo(w0.y), bf_hi(w0.y),
                                         bf_lo(w0.z), bf_hi(w0.z), bf_lo(w0.w), bf_hi(w0.w),
                                         bf_lo(w1.x), bf_hi(w1.x), bf_lo(w1.y), bf_hi(w1.y),
                                         bf_lo(w1.z), bf_hi(w1.z), bf_lo(w1.w), bf_hi(w1.w)};
#pragma unroll
                    for (int r = 0; r < kR; ++r)
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            o[r][e] = fmaf(prr[r], v[e], o[r][e]);
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
            if (lane == 0)
                mbar_arrive(&sm.empty[stage]);
        }
        T0 += ntiles;

        // --- combine the eight warp states of this item ---------------------
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
                    make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    *reinterpret_cast<float4 *>(&sm.wo[warp][r][h * 256 + lane * 8]) =
                        make_float4(o[r][h * 8 + 0], o[r][h * 8 + 1], o[r][h * 8 + 2],
                                    o[r][h * 8 + 3]);
                    *reinterpret_cast<float4 *>(&sm.wo[warp][r][h * 256 + lane * 8 + 4]) =
                        make_float4(o[r][h * 8 + 4], o[r][h * 8 + 5], o[r][h * 8 + 6],
                                    o[r][h * 8 + 7]);
                }
            }
        }
        named_barrier(1, kNCW * 32);
        // Element pairs of the kR x D block, dealt over the consumer threads.
        for (int e2 = warp * 32 + lane; e2 < kR * D / 2; e2 += kNCW * 32) {
            const int e0 = 2 * e2;
            const int r = e0 / D;
            const int col = e0 - r * D;
            const int m = it.b * kR + r;
            float mstar = NEG_INF;
#pragma unroll
            for (int w = 0; w < kNCW; ++w)
                mstar = fmaxf(mstar, sm.wm[w][r]);
            float lstar = 0.f, v0 = 0.f, v1 = 0.f;
#pragma unroll
            for (int w = 0; w < kNCW; ++w) {
                const float mw = sm.wm[w][r];
                const float wt = (mw == NEG_INF) ? 0.f : fast_exp2(mw - mstar);
                lstar = fmaf(sm.wl[w][r], wt, lstar);
                const float2 ov = *reinterpret_cast<const float2 *>(&sm.wo[w][r][col]);
                v0 = fmaf(ov.x, wt, v0);
                v1 = fmaf(ov.y, wt, v1);
            }
            if (m < p.M && !sm.abort_flag) {
                if (it.nc == 1) {
                    const int wr = m / p.G;
                    const int h = it.kh * p.G + (m - wr * p.G);
                    float *orow = p.out + (((size_t)it.s * p.W + wr) * p.Hq + h) * D;
                    const float inv = 1.f / lstar;
                    *reinterpret_cast<float2 *>(orow + col) = make_float2(v0 * inv, v1 * inv);
                } else {
                    float *slot = p.part + part_slot(p, it.s, it.kh, it.b, it.c) *
                                               (size_t)(p.RB * (D + 2));
                    *reinterpret_cast<float2 *>(slot + (size_t)r * D + col) = make_float2(v0, v1);
                    if (col == 0) {
                        slot[(size_t)p.RB * D + r] = mstar;
                        slot[(size_t)p.RB * D + p.RB + r] = lstar;
                    }
                }
            }
        }
        named_barrier(1, kNCW * 32);
    }
}

template <int D>
__global__ void __launch_bounds__(simt_threads<D>(), 1)
    attn_simt_kernel(const __grid_constant__ AttnParams p)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SimtSmem<D> &sm = *reinterpret_cast<SimtSmem<D> *>(smem_raw);
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < SimtSmem<D>::NSTAGE; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == SimtCfg<D>::NCW) {
        if (lane == 0)
            simt_producer<D>(p, sm);
        return;
    }
    simt_consumer<D>(p, sm, warp, lane);
}

// Host-side launcher (same translation unit as the kernel template).
template <int D>
cudaError_t launch_attn_simt(const AttnParams &p, int grid, cudaStream_t stream)
{
    const size_t smem = simt_smem_bytes<D>();
    static bool configured[kMaxDevices] = {};  // the attribute is set once per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(attn_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        configured[dev] = true;
    }
    attn_simt_kernel<D><<<grid, simt_threads<D>(), smem, stream>>>(p);
    return cudaGetLastError();
}

template cudaError_t launch_attn_simt<128>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_simt<512>(const AttnParams &, int, cudaStream_t);
template size_t simt_smem_bytes<128>();
template size_t simt_smem_bytes<512>();

}  // namespace tfp
