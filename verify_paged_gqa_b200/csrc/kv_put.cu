// kv_put.cu -- the row write: new K/V rows copied into their pages.
//
// TensorFold #1620, opening comment, "Writes": the rows kernel's new K and V
// rows are copied into the stream's pages.  Row r of stream s sits at
// position lens[s] - rows + r, i.e. in page table[s][pos / P], slot pos % P;
// for every KV head the head_dim bf16 values are copied bit for bit with
// 16-byte vector loads and stores.  One warp moves one (stream, row, KV head)
// row of K and V; rows whose length or page id is out of range are skipped.
#include "launch.cuh"

namespace tfp {

__global__ void __launch_bounds__(256) kv_put_kernel(const __grid_constant__ PutParams p)
{
    allow_dependent_launch();  // the attention kernel after it may be scheduled now
    const int warps = blockDim.x / 32;
    const int64_t row = (int64_t)blockIdx.x * warps + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int64_t total = (int64_t)p.S * p.W * p.Hkv;
    if (row >= total)
        return;
    const int kh = static_cast<int>(row % p.Hkv);
    const int64_t sr = row / p.Hkv;
    const int r = static_cast<int>(sr % p.W);
    const int s = static_cast<int>(sr / p.W);
    const int len = __ldg(p.lens + s);
    if (len < p.W || (int64_t)len > (int64_t)p.table_stride * p.P)
        return;
    const int pos = len - p.W + r;
    const int lp = pos / p.P;
    const int page = __ldg(p.table + (int64_t)s * p.table_stride + lp);
    if (page < 0 || page >= p.n_pages)
        return;
    const size_t dst = (((size_t)page * p.Hkv + kh) * p.P + (pos - lp * p.P)) * p.D;
    const size_t src = (size_t)row * p.D;
    const int nvec = p.D / 8;  // 16-byte vectors per row
    const uint4 *ks = reinterpret_cast<const uint4 *>(p.k_rows + src);
    const uint4 *vs = reinterpret_cast<const uint4 *>(p.v_rows + src);
    uint4 *kd = reinterpret_cast<uint4 *>(p.k_pool + dst);
    uint4 *vd = reinterpret_cast<uint4 *>(p.v_pool + dst);
    for (int i = lane; i < 2 * nvec; i += 32) {
        if (i < nvec)
            kd[i] = __ldg(ks + i);
        else
            vd[i - nvec] = __ldg(vs + (i - nvec));
    }
}

cudaError_t launch_kv_put(const PutParams &p, cudaStream_t stream)
{
    const int64_t rows = (int64_t)p.S * p.W * p.Hkv;
    if (rows == 0)
        return cudaSuccess;
    const int warps = 8;
    const int64_t blocks = (rows + warps - 1) / warps;
    kv_put_kernel<<<static_cast<unsigned>(blocks), warps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tfp
