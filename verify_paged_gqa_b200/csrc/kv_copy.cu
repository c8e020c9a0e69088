// kv_copy.cu -- the state copy: a stream's K/V walked from one set of pages
// to another.
//
// TensorFold #1620, opening comment, "Kept states" bullet: a kept state is
// copied by walking the slot's pages.  For every stream s, position
// j < lens[s] and KV head kh, the head_dim bf16 values of K and of V move bit
// for bit from source page src_table[s][j / Ps], slot j % Ps, to destination
// page dst_table[s][j / Pd], slot j % Pd.  A linear buffer is a pool with one
// page per stream, so keeping a state, resuming it and reusing pages are all
// this copy.
//
// One block (one issuing lane) per chunk of CH positions of one (stream, KV
// head), CH * head_dim * 2 = 16 KB per tensor: bulk copies (TMA engine) of
// the chunk's source page pieces into shared memory, completing on one
// mbarrier, then bulk stores of its destination page pieces out of it.
// Several blocks share an SM, so their loads and stores overlap.  A piece on
// a page outside its pool is not read or written and sets TF_DEV_BAD_PAGE; a
// stream whose length is out of range is skipped and sets TF_DEV_BAD_LEN.
#include "launch.cuh"

namespace tfp {

namespace {

constexpr uint32_t kChunkBytes = 16384;  // per tensor (K or V) per block

__device__ __forceinline__ void copy_flag(uint32_t *status, uint32_t bit)
{
    if (status)
        atomicOr(status, bit);
}

__global__ void __launch_bounds__(32) kv_copy_kernel(const __grid_constant__ CopyParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];  // K rows, then V rows
    __shared__ uint64_t bar;
    if (threadIdx.x != 0)
        return;
    const int64_t b = blockIdx.x;
    const int c = static_cast<int>(b % p.n_chunks);
    const int64_t sk = b / p.n_chunks;
    const int kh = static_cast<int>(sk % p.Hkv);
    const int s = static_cast<int>(sk / p.Hkv);
    const int len = __ldg(p.lens + s);
    if (len < 0 || len > p.max_len || (int64_t)len > (int64_t)p.src_stride * p.src_P ||
        (int64_t)len > (int64_t)p.dst_stride * p.dst_P) {
        if (c == 0 && kh == 0)
            copy_flag(p.status, kDevBadLen);
        return;
    }
    const int p0 = c * p.chunk;
    if (p0 >= len)
        return;
    const int p1 = min(p0 + p.chunk, len);
    const uint32_t row = static_cast<uint32_t>(p.D) * 2u;
    uint8_t *vs = smem + static_cast<size_t>(p.chunk) * row;
    const uint64_t pol = l2_evict_first_policy();

    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, 2u * static_cast<uint32_t>(p1 - p0) * row);
    // the source pieces: one bulk copy of K and one of V per page run
    const int32_t *strow = p.src_table + (int64_t)s * p.src_stride;
    for (int pos = p0; pos < p1;) {
        const int lp = pos / p.src_P;
        const int n = min((lp + 1) * p.src_P, p1) - pos;
        const int32_t page = __ldg(strow + lp);
        const uint32_t nb = static_cast<uint32_t>(n) * row;
        if (page >= 0 && page < p.src_n_pages) {
            const size_t off = (((size_t)page * p.Hkv + kh) * p.src_P + (pos - lp * p.src_P)) * p.D;
            bulk_g2s(smem + (size_t)(pos - p0) * row, p.src_k + off, nb, &bar, pol);
            bulk_g2s(vs + (size_t)(pos - p0) * row, p.src_v + off, nb, &bar, pol);
        } else {
            copy_flag(p.status, kDevBadPage);
            mbar_complete_tx(&bar, 2u * nb);
        }
        pos += n;
    }
    if (!mbar_wait(&bar, 0)) {
        copy_flag(p.status, kDevTimeout);
        (void)mbar_wait(&bar, 0);  // the copies in flight land before the block exits
        return;
    }
    // the destination pieces
    const int32_t *dtrow = p.dst_table + (int64_t)s * p.dst_stride;
    for (int pos = p0; pos < p1;) {
        const int lp = pos / p.dst_P;
        const int n = min((lp + 1) * p.dst_P, p1) - pos;
        const int32_t page = __ldg(dtrow + lp);
        const uint32_t nb = static_cast<uint32_t>(n) * row;
        if (page >= 0 && page < p.dst_n_pages) {
            const size_t off = (((size_t)page * p.Hkv + kh) * p.dst_P + (pos - lp * p.dst_P)) * p.D;
            bulk_s2g(p.dst_k + off, smem + (size_t)(pos - p0) * row, nb);
            bulk_s2g(p.dst_v + off, vs + (size_t)(pos - p0) * row, nb);
        } else {
            copy_flag(p.status, kDevBadPage);
        }
        pos += n;
    }
    bulk_commit();
    bulk_wait_all();
}

}  // namespace

int copy_chunk_positions(int head_dim)
{
    return static_cast<int>(kChunkBytes / (static_cast<uint32_t>(head_dim) * 2u));
}

cudaError_t launch_kv_copy(const CopyParams &p, cudaStream_t stream)
{
    const int64_t blocks = (int64_t)p.S * p.Hkv * p.n_chunks;
    if (blocks == 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidValue;
    const size_t bytes = 2u * kChunkBytes;
    kv_copy_kernel<<<static_cast<unsigned>(blocks), 32, bytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tfp
