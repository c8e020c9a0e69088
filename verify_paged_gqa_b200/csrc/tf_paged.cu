// tf_paged.cu -- the C ABI: argument checks, the launch plan, dispatch.
//
// Every entry point checks its host arguments before enqueueing anything
// and returns a TF_* status.  The plan (row blocks, context chunk, grid)
// depends only on host arguments and the device's SM count, so a captured
// graph stays valid while lens grow up to max_len.
#include "../../include/tf_paged.h"
#include "../../include/tf_paged_testing.h"
#include "launch.cuh"
#include "plan.cuh"

#include <atomic>
#include <cmath>
#include <mutex>

namespace tfp {
namespace {

// The SM count of the current device, queried once per device.  Host threads
// making their first calls at once may each query it and store the same
// value; the atomics keep that race well defined.
int device_sm_count(int *sms)
{
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return TF_ECUDA;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            n <= 0)
            return TF_ECUDA;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    *sms = n;
    return TF_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_pool_streams(const tf_kv_pool *pool, const tf_streams *st)
{
    if (!pool || !st)
        return TF_EINVAL;
    if (pool->n_pages < 1 || pool->n_kv_heads < 1 || pool->page_size < 1)
        return TF_EINVAL;
    if (pool->head_dim != 128 && pool->head_dim != 256 && pool->head_dim != 512)
        return TF_EUNSUPPORTED;
    if (st->n_streams < 0 || st->table_stride < 1 || st->max_len < 1)
        return TF_EINVAL;
    if ((int64_t)st->max_len > (int64_t)st->table_stride * pool->page_size)
        return TF_EINVAL;
    if ((int64_t)st->n_streams * st->table_stride > INT32_MAX)
        return TF_EINVAL;
    if (st->n_streams > 0 && (!st->table || !st->lens))
        return TF_EINVAL;
    if (!pool->k_pool || !pool->v_pool || !aligned16(pool->k_pool) || !aligned16(pool->v_pool))
        return TF_EINVAL;
    return TF_OK;
}

enum class Kernel { kSimt, kPrompt, kPm };

// Workspace: the 256-byte header (status word, wait site, the launch's tile
// count at byte 64), each stream's first tile (int64), then two partial slots
// per CTA of min(RB, M) rows x (D + 2) floats (rounded up to 16 bytes).
constexpr size_t kWsTotalOffset = 64;

size_t ws_part_offset(int S)
{
    return kWsHeaderBytes + (((size_t)S * 8 + 255) / 256) * 256;
}

// Entry tiles per unit (plan.cuh), measured: at head dim 512 a unit start
// costs about 8 tiles' worth of streaming (the ring holds less than one
// tile, so the pipeline drains and refills); the prompt kernel's split
// units (more than 64 rows per KV head over long contexts) pay its serial
// epilogue and its query load, about 8 of its tiles; the CUDA-core decode
// kernel's segment starts overlap with its deep ring and cost nothing
// measurable.
constexpr int kEntryPm512 = 8;
constexpr int kEntryPm128 = 6;
constexpr int kEntryPrompt = 8;
constexpr int kEntrySimt = 0;

// Decode blocks at head dim 128 take the position-major kernel from this
// max_len on (measured crossover near 5,700 positions).
constexpr int kPmDecodeMinLen = 6144;

struct Plan {
    AttnParams p;
    int grid;
    size_t ws_bytes;
    Kernel kernel;  // which partial kernel runs the call
};

int make_plan(const tf_kv_pool *pool, const tf_streams *st, int32_t Hq, int32_t rows,
              int32_t rows_max, bool tree, Plan *plan)
{
    int rc = check_pool_streams(pool, st);
    if (rc != TF_OK)
        return rc;
    if (Hq < 1 || Hq % pool->n_kv_heads != 0)
        return TF_EINVAL;
    if (rows < 1 || rows > rows_max || st->max_len < rows)
        return TF_EINVAL;
    const int G = Hq / pool->n_kv_heads;
    const int64_t M = (int64_t)G * rows;
    if (M > (1 << 20))
        return TF_EINVAL;
    int sms = 0;
    rc = device_sm_count(&sms);
    if (rc != TF_OK)
        return rc;

    AttnParams &p = plan->p;
    p = AttnParams{};
    p.n_pages = pool->n_pages;
    p.Hkv = pool->n_kv_heads;
    p.P = pool->page_size;
    p.D = pool->head_dim;
    p.table_stride = st->table_stride;
    p.S = st->n_streams;
    p.max_len = st->max_len;
    p.Hq = Hq;
    p.G = G;
    p.W = rows;
    p.M = static_cast<int32_t>(M);
    p.has_tree = tree ? 1 : 0;
    p.withhold = 0;
    p.wait_limit = kWaitLimitCycles;
    // Rows sharing a KV head go to the tensor cores as a dense QK^T / PV
    // tile: up to 64 rows (any count at head dims 256 and 512, in blocks of
    // 32) with the positions on the MMA's M, larger blocks with the rows
    // there.  At head dim 128 that holds for a single CUDA-core row block
    // too (decode at GQA 4): its two MMA issuers keep pace with HBM at any
    // clock, where the CUDA-core kernel's FMAs fall behind under the power
    // cap (12 x 40,960 decode: 341 -> 296 us per call).  Head dim 512 keeps
    // such calls on the CUDA-core kernel.  Pages that are not a multiple of
    // 128 positions: the tensor-core kernels assemble each tile from page
    // pieces, one TMA box per set bit of a piece's length, so small pages
    // cost many box loads per tile.  For a single 4-row block (decode at
    // GQA <= 4) the CUDA-core kernel, which copies pieces into its own
    // smaller tiles, is then faster below 128 positions unless the page is a
    // multiple of 64 (12 x 40,960 decode, GB/s, CUDA-core / tensor-core:
    // pages of 37 3,378 / 1,915; 48 3,995 / 3,175; 64 5,045 / 5,190; 96
    // 5,368 / 4,830; 100 4,208 / 3,599; 200 4,555 / 4,951; 509 4,697 /
    // 5,527).  Several row blocks would each re-read the K/V on the CUDA-core
    // kernel, so larger blocks always take the tensor cores (verify
    // 4 x 131,072 in pages of 64: 311 against 4,467 GB/s).  Pools past 2^31
    // rows run on the CUDA-core kernel.
    const bool small_odd_pages = p.P < 128 && p.P % 64 != 0;
    // A decode block also stays on the CUDA-core kernel for short contexts:
    // the position-major kernel pays about six tiles (768 positions) to start
    // each (stream, KV head) unit, which outweighs its steady-state lead
    // below about 6,000 positions (GB/s, position-major / CUDA-core: 64 x
    // 2,048 4,507 / 5,112; 256 x 512 3,207 / 3,638; 12 x 8,192 5,315 /
    // 5,187; 12 x 40,960 6,875 / 6,061).  max_len bounds every stream, so the
    // choice depends on host arguments only.
    const bool long_context = st->max_len >= kPmDecodeMinLen;
    plan->kernel = Kernel::kSimt;
    p.RB = kSimtRows;
    if (tree) {
        // tree masks: the position-major kernel (any row count), else the
        // CUDA-core kernel (pools past 2^31 rows)
        const int nr = pm_rows(p);
        if (nr > 0) {
            plan->kernel = Kernel::kPm;
            p.RB = nr;
        } else if (p.D == 256) {
            return TF_EUNSUPPORTED;
        }
    } else if (p.D == 256) {
        // head dim 256 runs on the position-major kernel only (any row count)
        const int nr = pm_rows(p);
        if (nr == 0)
            return TF_EUNSUPPORTED;
        plan->kernel = Kernel::kPm;
        p.RB = nr;
    } else if (M > kSimtRows || (p.D == 128 && !small_odd_pages && long_context)) {
        const int nr = pm_rows(p);
        if (nr > 0) {
            plan->kernel = Kernel::kPm;
            p.RB = nr;
        } else if (prompt_supported(p)) {
            plan->kernel = Kernel::kPrompt;
            p.RB = prompt_rows();
        }
    }
    p.n_rblk = static_cast<int32_t>((M + p.RB - 1) / p.RB);
    p.SR = static_cast<int32_t>(M < p.RB ? M : p.RB);

    // Entry cost of a unit, in tiles: what starting one more unit costs a
    // CTA relative to streaming one tile of it (measured per kernel).
    p.VT = plan->kernel == Kernel::kPm ? (p.D == 512 ? kEntryPm512 : kEntryPm128)
         : plan->kernel == Kernel::kPrompt ? kEntryPrompt : kEntrySimt;
    // One persistent CTA per SM, but no more than the work the call can have
    // with every stream at max_len (the device splits the actual work).
    const int64_t tiles_max = (int64_t)p.S * p.Hkv * head_work(p, st->max_len);
    int64_t grid = sms < kMaxCtas ? sms : kMaxCtas;
    if (tiles_max < grid)
        grid = tiles_max > 0 ? tiles_max : 1;
    // A tensor-bound prompt call whose units fill most CTAs (but no more)
    // gives each CTA one whole unit: the split's partials and merge cost more
    // than a few idle SMs (measured on the chunked prompt: 128 units on 148).
    const int64_t units = (int64_t)p.S * p.Hkv * p.n_rblk;
    const int cap = sms < kMaxCtas ? sms : kMaxCtas;
    p.whole = plan->kernel == Kernel::kPrompt && units <= cap && 4 * units >= 3 * (int64_t)cap;
    if (p.whole)
        grid = units > 0 ? units : 1;
    plan->grid = static_cast<int>(grid);
    p.n_cta = plan->grid;
    plan->ws_bytes = ws_part_offset(p.S) + (size_t)2 * plan->grid * part_slot_floats(p) * sizeof(float);
    return TF_OK;
}

// The test hooks of one call (tf_testing_paged_attn); none in library calls.
struct Faults {
    long long wait_limit = kWaitLimitCycles;
    int32_t withhold = 0;
};

int attn_call(const tf_kv_pool *pool, const tf_streams *st, const void *q, int32_t Hq,
              int32_t rows, int32_t rows_max, const uint8_t *tree, float scale, float *out,
              void *ws, size_t ws_bytes, void *stream, const Faults &faults = Faults{})
{
    Plan plan;
    int rc = make_plan(pool, st, Hq, rows, rows_max, tree != nullptr, &plan);
    if (rc != TF_OK)
        return rc;
    plan.p.wait_limit = faults.wait_limit;
    plan.p.withhold = faults.withhold;
    if (!std::isfinite(scale))
        return TF_EINVAL;
    if (st->n_streams == 0)
        return TF_OK;  // nothing is read or written: the buffers may be null
    if (!q || !out || !ws || !aligned16(q) || !aligned16(out) || !aligned16(ws))
        return TF_EINVAL;
    if (ws_bytes < plan.ws_bytes)
        return TF_ENOSPACE;
    AttnParams &p = plan.p;
    p.k_pool = static_cast<const __nv_bfloat16 *>(pool->k_pool);
    p.v_pool = static_cast<const __nv_bfloat16 *>(pool->v_pool);
    p.table = st->table;
    p.lens = st->lens;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.tree = tree;
    p.out = out;
    char *wsb = static_cast<char *>(ws);
    p.flags = reinterpret_cast<uint32_t *>(wsb);
    p.total_tiles = reinterpret_cast<long long *>(wsb + kWsTotalOffset);
    p.first_tile = reinterpret_cast<long long *>(wsb + kWsHeaderBytes);
    p.part = reinterpret_cast<float *>(wsb + ws_part_offset(p.S));
    p.scale_log2 = scale * 1.4426950408889634f;  // log2(e)
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (plan.kernel == Kernel::kPm) {
        e = launch_attn_pm(p, plan.grid, s);
        if (e == cudaSuccess)
            e = p.D == 128   ? launch_attn_merge<128>(p, s)
                : p.D == 256 ? launch_attn_merge<256>(p, s)
                             : launch_attn_merge<512>(p, s);
    } else if (plan.kernel == Kernel::kPrompt) {
        e = launch_attn_prompt(p, plan.grid, s);
        if (e == cudaSuccess)
            e = launch_attn_merge<128>(p, s);
    } else if (p.D == 128) {
        e = launch_attn_simt<128>(p, plan.grid, s);
        if (e == cudaSuccess)
            e = launch_attn_merge<128>(p, s);
    } else {
        e = launch_attn_simt<512>(p, plan.grid, s);
        if (e == cudaSuccess)
            e = launch_attn_merge<512>(p, s);
    }
    return e == cudaSuccess ? TF_OK : TF_ECUDA;
}

}  // namespace
}  // namespace tfp

using namespace tfp;

extern "C" {

int tf_kv_put_rows(const tf_kv_pool *pool, const tf_streams *streams, const void *k_rows,
                   const void *v_rows, int32_t rows, void *stream)
{
    int rc = check_pool_streams(pool, streams);
    if (rc != TF_OK)
        return rc;
    if (rows < 1 || streams->max_len < rows)
        return TF_EINVAL;
    if (streams->n_streams == 0)
        return TF_OK;
    if (!k_rows || !v_rows || !aligned16(k_rows) || !aligned16(v_rows))
        return TF_EINVAL;
    PutParams p;
    p.k_pool = static_cast<__nv_bfloat16 *>(pool->k_pool);
    p.v_pool = static_cast<__nv_bfloat16 *>(pool->v_pool);
    p.table = streams->table;
    p.lens = streams->lens;
    p.k_rows = static_cast<const __nv_bfloat16 *>(k_rows);
    p.v_rows = static_cast<const __nv_bfloat16 *>(v_rows);
    p.n_pages = pool->n_pages;
    p.Hkv = pool->n_kv_heads;
    p.P = pool->page_size;
    p.D = pool->head_dim;
    p.table_stride = streams->table_stride;
    p.S = streams->n_streams;
    p.W = rows;
    return launch_kv_put(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TF_OK : TF_ECUDA;
}

int tf_kv_copy_state(const tf_kv_pool *src_pool, const tf_streams *src,
                     const tf_kv_pool *dst_pool, const int32_t *dst_table,
                     int32_t dst_table_stride, uint32_t *status, void *stream)
{
    int rc = check_pool_streams(src_pool, src);
    if (rc != TF_OK)
        return rc;
    if (!dst_pool || dst_pool->n_pages < 1 || dst_pool->page_size < 1)
        return TF_EINVAL;
    if (dst_pool->n_kv_heads != src_pool->n_kv_heads || dst_pool->head_dim != src_pool->head_dim)
        return TF_EINVAL;
    if (!dst_pool->k_pool || !dst_pool->v_pool || !aligned16(dst_pool->k_pool) ||
        !aligned16(dst_pool->v_pool))
        return TF_EINVAL;
    if (dst_table_stride < 1 ||
        (int64_t)src->max_len > (int64_t)dst_table_stride * dst_pool->page_size ||
        (int64_t)src->n_streams * dst_table_stride > INT32_MAX)
        return TF_EINVAL;
    if (src->n_streams > 0 && !dst_table)
        return TF_EINVAL;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u) != 0)
        return TF_EINVAL;
    if (src->n_streams == 0)
        return TF_OK;
    CopyParams p;
    p.src_k = static_cast<const __nv_bfloat16 *>(src_pool->k_pool);
    p.src_v = static_cast<const __nv_bfloat16 *>(src_pool->v_pool);
    p.dst_k = static_cast<__nv_bfloat16 *>(dst_pool->k_pool);
    p.dst_v = static_cast<__nv_bfloat16 *>(dst_pool->v_pool);
    p.src_table = src->table;
    p.dst_table = dst_table;
    p.lens = src->lens;
    p.status = status;
    p.src_stride = src->table_stride;
    p.dst_stride = dst_table_stride;
    p.src_P = src_pool->page_size;
    p.dst_P = dst_pool->page_size;
    p.src_n_pages = src_pool->n_pages;
    p.dst_n_pages = dst_pool->n_pages;
    p.Hkv = src_pool->n_kv_heads;
    p.D = src_pool->head_dim;
    p.S = src->n_streams;
    p.max_len = src->max_len;
    p.chunk = copy_chunk_positions(p.D);
    p.n_chunks = (src->max_len + p.chunk - 1) / p.chunk;
    return launch_kv_copy(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TF_OK : TF_ECUDA;
}

size_t tf_paged_attn_workspace_bytes(const tf_kv_pool *pool, const tf_streams *streams,
                                     int32_t n_q_heads, int32_t rows)
{
    Plan plan;
    if (make_plan(pool, streams, n_q_heads, rows, 4096, false, &plan) != TF_OK)
        return 0;
    size_t bytes = plan.ws_bytes;
    // enough for a tree-verify call with the same arguments too
    Plan tp;
    if (rows <= 8 && make_plan(pool, streams, n_q_heads, rows, 8, true, &tp) == TF_OK &&
        tp.ws_bytes > bytes)
        bytes = tp.ws_bytes;
    return bytes;
}

int tf_paged_attn_decode(const tf_kv_pool *pool, const tf_streams *streams, const void *q,
                         int32_t n_q_heads, float scale, float *out, void *workspace,
                         size_t workspace_bytes, void *stream)
{
    return attn_call(pool, streams, q, n_q_heads, 1, 1, nullptr, scale, out, workspace,
                     workspace_bytes, stream);
}

int tf_paged_attn_verify(const tf_kv_pool *pool, const tf_streams *streams, const void *q,
                         int32_t n_q_heads, int32_t rows, float scale, float *out,
                         void *workspace, size_t workspace_bytes, void *stream)
{
    return attn_call(pool, streams, q, n_q_heads, rows, 8, nullptr, scale, out, workspace,
                     workspace_bytes, stream);
}

int tf_paged_attn_verify_tree(const tf_kv_pool *pool, const tf_streams *streams, const void *q,
                              int32_t n_q_heads, int32_t rows, const uint8_t *tree_masks,
                              float scale, float *out, void *workspace, size_t workspace_bytes,
                              void *stream)
{
    if (streams && streams->n_streams > 0 && !tree_masks)
        return TF_EINVAL;
    return attn_call(pool, streams, q, n_q_heads, rows, 8, tree_masks, scale, out, workspace,
                     workspace_bytes, stream);
}

int tf_paged_attn_prompt(const tf_kv_pool *pool, const tf_streams *streams, const void *q,
                         int32_t n_q_heads, int32_t rows, float scale, float *out,
                         void *workspace, size_t workspace_bytes, void *stream)
{
    return attn_call(pool, streams, q, n_q_heads, rows, 4096, nullptr, scale, out, workspace,
                     workspace_bytes, stream);
}

int tf_testing_paged_attn(const tf_kv_pool *pool, const tf_streams *streams, const void *q,
                          int32_t n_q_heads, int32_t rows, float scale, float *out,
                          void *workspace, size_t workspace_bytes, int64_t wait_limit_cycles,
                          int32_t withhold, void *stream)
{
    if (wait_limit_cycles < 1000000 || wait_limit_cycles > kWaitLimitCycles)
        return TF_EINVAL;
    if (withhold != 0 && withhold != 1)
        return TF_EINVAL;
    Faults f;
    f.wait_limit = wait_limit_cycles;
    f.withhold = withhold;
    return attn_call(pool, streams, q, n_q_heads, rows, 4096, nullptr, scale, out, workspace,
                     workspace_bytes, stream, f);
}

int tf_workspace_status(void *workspace, uint32_t *flags, void *stream)
{
    if (!workspace || !flags)
        return TF_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t host = 0;
    if (cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return TF_ECUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof host, s) != cudaSuccess)
        return TF_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return TF_ECUDA;
    *flags = host;
    return TF_OK;
}

const char *tf_status_str(int status)
{
    switch (status) {
    case TF_OK:
        return "TF_OK";
    case TF_EINVAL:
        return "TF_EINVAL: invalid argument";
    case TF_EUNSUPPORTED:
        return "TF_EUNSUPPORTED: shape not supported by this library";
    case TF_ENOSPACE:
        return "TF_ENOSPACE: workspace too small";
    case TF_ECUDA:
        return "TF_ECUDA: CUDA launch or query failed";
    default:
        return "unknown status";
    }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without a caller-provided workspace.
//
// Some callers cannot allocate device memory for a workspace: a plug-in
// hosted by an inference engine that hands it only its input and output
// buffers and owns every allocation itself, or a serving loop that must not
// call cudaMalloc once it is running (cudaMalloc can synchronise the device
// and can fail under memory pressure).  For them the split-context scratch
// lives in one file-scope device array of kStaticScratchBytes, which every
// GPU that loads this library keeps until the process exits.
namespace tfp {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so its device address is
// looked up once per device (with that device current) and cached.
int static_scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return TF_ECUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
            return TF_ECUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return TF_OK;
}

}  // namespace
}  // namespace tfp

extern "C" int tf_paged_attn_decode_noalloc(const tf_kv_pool *pool, const tf_streams *streams,
                                            const void *q, int32_t n_q_heads, float scale,
                                            float *out, void *stream)
{
    using namespace tfp;
    Plan plan;
    int rc = make_plan(pool, streams, n_q_heads, 1, 1, false, &plan);
    if (rc != TF_OK)
        return rc;
    if (!std::isfinite(scale))
        return TF_EINVAL;
    // as tf_paged_attn_decode: a call with no streams reads and writes
    // nothing, and its buffers may be null
    if (streams->n_streams == 0)
        return TF_OK;
    if (!q || !out || !aligned16(q) || !aligned16(out))
        return TF_EINVAL;
    if (plan.ws_bytes > kStaticScratchBytes)
        return TF_ENOSPACE;
    void *ws = nullptr;
    rc = static_scratch_address(&ws);
    if (rc != TF_OK)
        return rc;
    // Nothing in the scratch needs clearing: the kernels write every partial
    // and the header's tile counts before reading them.  The header's status
    // and wait-site words only collect bits (ORed in by the kernels) that no
    // kernel reads and this call does not report, so they are left as they
    // are; their contents are unspecified.
    return attn_call(pool, streams, q, n_q_heads, 1, 1, nullptr, scale, out, ws, kStaticScratchBytes,
                     stream);
}
