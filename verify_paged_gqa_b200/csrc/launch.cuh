// launch.cuh -- host-side launchers of the kernels (one per translation unit).
#pragma once

#include "common.cuh"

#include <atomic>

namespace tfp {

// Raises `kernel`'s dynamic shared memory limit to `bytes`, once per device
// (done[dev] records it).  Host threads making their first launches at once
// may each set the same attribute, which is harmless; the flags are atomics,
// so that race is well defined.
template <class Kernel>
cudaError_t set_smem_limit_once(Kernel kernel, size_t bytes, std::atomic<bool> (&done)[kMaxDevices])
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire))
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess)
        done[dev].store(true, std::memory_order_release);
    return e;
}

// Launches `kernel` as a programmatic dependent of the previous kernel in the
// stream: its blocks may be scheduled while that kernel finishes, and wait
// for it in the kernel (wait_prior_grid) before reading its outputs.
template <class Kernel, class Arg>
cudaError_t launch_dependent(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             const Arg &arg)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, arg);
}

struct PutParams {
    __nv_bfloat16 *k_pool;
    __nv_bfloat16 *v_pool;
    const int32_t *table;
    const int32_t *lens;
    const __nv_bfloat16 *k_rows;
    const __nv_bfloat16 *v_rows;
    int32_t n_pages, Hkv, P, D;
    int32_t table_stride, S, W;
};

cudaError_t launch_kv_put(const PutParams &p, cudaStream_t stream);

// The state copy (kv_copy.cu): positions [0, lens[s]) of every KV head from
// the source pool's pages to the destination pool's pages.
struct CopyParams {
    const __nv_bfloat16 *src_k;
    const __nv_bfloat16 *src_v;
    __nv_bfloat16 *dst_k;
    __nv_bfloat16 *dst_v;
    const int32_t *src_table;
    const int32_t *dst_table;
    const int32_t *lens;
    uint32_t *status;              // TF_DEV_* bits are ORed in (may be null)
    int32_t src_stride, dst_stride, src_P, dst_P, src_n_pages, dst_n_pages;
    int32_t Hkv, D, S, max_len;
    int32_t chunk;                 // positions per block
    int32_t n_chunks;              // blocks per (stream, KV head): ceil(max_len / chunk)
};

int copy_chunk_positions(int head_dim);
cudaError_t launch_kv_copy(const CopyParams &p, cudaStream_t stream);

// Rows per row block of the CUDA-core partial kernel.
constexpr int kSimtRows = 4;

template <int D>
size_t simt_smem_bytes();
template <int D>
cudaError_t launch_attn_simt(const AttnParams &p, int grid, cudaStream_t stream);
template <int D>
cudaError_t launch_attn_merge(const AttnParams &p, cudaStream_t stream);  // D 128, 256, 512

// Prompt tensor-core partial kernel (tcgen05): row blocks of prompt_rows()
// rows on the QK MMA's M, PV transposed.
int prompt_rows();
bool prompt_supported(const AttnParams &p);
cudaError_t launch_attn_prompt(const AttnParams &p, int grid, cudaStream_t stream);

// Position-major tensor-core partial kernel: key positions on the MMA's M,
// row blocks of pm_rows(p) rows (0: not supported for these arguments).
int pm_rows(const AttnParams &p);
cudaError_t launch_attn_pm(const AttnParams &p, int grid, cudaStream_t stream);

}  // namespace tfp
