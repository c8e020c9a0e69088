/*
 * tf_paged.h -- attention over a paged KV cache on NVIDIA B200 (sm_100a).
 *
 * Keys and values live in fixed pages of `page_size` positions drawn from
 * one shared pool; every stream reads its positions through its own row of
 * a page table.  The library provides the row write that copies new K/V rows
 * into their pages, and grouped-query attention for single-row decode,
 * draft-verify windows (causal inside the window) and chunked prompt rows.
 *
 * Sources (the TensorFold pull-request pages this library follows):
 *  - TensorFold #1620, "Kolibri-1's full layers take their K/V from pages of
 *    the core pool", opening comment:
 *      * "Pages of 512 positions": the pool and its fixed page size;
 *      * "Writes": new K/V rows are copied into the pages (tf_kv_put_rows);
 *      * "Reads": prompt rows, decode and drafted verify read keys through a
 *        page table given in the call's stream order (the tf_paged_attn_*
 *        calls);
 *    and its later comment on per-tile page lookup: a tile's page is looked
 *    up once per tile, and paging leaves the result bits unchanged.
 *  - TensorFold #2730, "an eight-row verify window", section "What this
 *    changes": a verify window is the pending token plus up to seven drafts.
 *
 * Conventions shared by every call
 * --------------------------------
 *  Layouts (all row-major, element counts, no padding):
 *    K pool, V pool  bf16  [n_pages][n_kv_heads][page_size][head_dim]  device
 *    table           int32 [n_streams][table_stride]                   device
 *    lens            int32 [n_streams]                                  device
 *    q               bf16  [n_streams][rows][n_q_heads][head_dim]       device
 *    out             fp32  [n_streams][rows][n_q_heads][head_dim]       device
 *    k_rows, v_rows  bf16  [n_streams][rows][n_kv_heads][head_dim]      device
 *
 *  lens[s] counts the positions of stream s AFTER this step's rows are
 *  written.  Window row r (0 <= r < rows) sits at position
 *  lens[s] - rows + r and attends to positions 0 .. lens[s] - rows + r.
 *  Position j of stream s lives in pool page table[s][j / page_size], slot
 *  j % page_size.  Query head h reads KV head h / (n_q_heads / n_kv_heads).
 *
 *  The output is softmax(scale * q . k) weighted sum of v, accumulated in
 *  fp32 from bf16 inputs.  Which pool pages hold a stream's positions never
 *  changes a bit of the result: the arithmetic depends only on positions,
 *  lens, rows and the host arguments.
 *
 *  Ownership: the caller owns every buffer.  The library allocates nothing
 *  and keeps no state between calls; each call enqueues kernels on the
 *  caller's CUDA stream (`stream` is a cudaStream_t; NULL is the legacy
 *  default stream) and returns without waiting.
 *
 *  Errors: every call checks its host arguments before enqueueing anything
 *  and returns a TF_* status; on a non-zero status nothing was enqueued
 *  (TF_ECUDA: a launch failed).  lens and table are device data and are
 *  checked on the device: a stream whose length is outside
 *  [rows, min(max_len, table_stride * page_size)] is skipped and its
 *  outputs are set to NaN; a page id outside [0, n_pages) is never read.
 *  Such events set bits in the workspace's status word (tf_workspace_status).
 *  Table entries past ceil(lens[s] / page_size) are never read, and pool
 *  slots at or past lens[s] never reach an output, whatever they hold.
 *
 *  Graph capture: lens and table are read on the device, and max_len only
 *  bounds the launch, so one captured graph serves growing lengths up to
 *  max_len.
 */
#ifndef TF_PAGED_H
#define TF_PAGED_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TF_API __attribute__((visibility("default")))
#else
#define TF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call. */
#define TF_OK 0
#define TF_EINVAL 1        /* a NULL pointer, a bad size or an inconsistent shape */
#define TF_EUNSUPPORTED 2  /* a shape this library has no kernel for (head_dim, page_size) */
#define TF_ENOSPACE 3      /* the workspace is smaller than tf_paged_attn_workspace_bytes */
#define TF_ECUDA 4         /* a CUDA launch or query failed */

/* Bits of the device-side status word (tf_workspace_status). */
#define TF_DEV_BAD_LEN 1u   /* some lens[s] outside [rows, min(max_len, table_stride*page_size)] */
#define TF_DEV_BAD_PAGE 2u  /* some table entry in use outside [0, n_pages) */
#define TF_DEV_TIMEOUT 4u   /* a pipeline wait gave up (an internal error) */

/* The pool: K and V pages, device memory, 16-byte aligned.
 * page_size may be any positive size at every head dim (TensorFold #1620,
 * Checks, the kernel-contract bullet: the paged prompt kernel is checked
 * over pages of 512, 37 and 64); head_dim must be 128, 256 or 512.  Pages
 * that are not a multiple of 128 positions are read by tiles assembled from
 * page pieces; the results do not depend on the page size.  Head dim 256
 * calls are refused (TF_EUNSUPPORTED) for pools of more than 2^31 - 1 rows
 * (n_pages * n_kv_heads * page_size). */
typedef struct tf_kv_pool {
    void *k_pool;
    void *v_pool;
    int32_t n_pages;
    int32_t n_kv_heads;
    int32_t page_size;
    int32_t head_dim;
} tf_kv_pool;

/* The streams of one call: page table, lengths (device) and a host upper
 * bound on the lengths.  max_len <= table_stride * page_size. */
typedef struct tf_streams {
    const int32_t *table;
    int32_t table_stride;
    const int32_t *lens;
    int32_t n_streams;  /* 0: every call checks its host arguments, then does
                         * nothing and returns TF_OK (its buffers may be null) */
    int32_t max_len;
} tf_streams;

/* Row write (TensorFold #1620, opening comment, "Writes").
 * Copies `rows` new K and V rows per stream into their pages: row r of
 * stream s (k_rows[s][r][kh][:]) goes to position lens[s] - rows + r.  The
 * copy is bitwise; nothing else in the pool is touched.  A row whose
 * stream length or page id is out of range is skipped.  rows >= 1. */
TF_API int tf_kv_put_rows(const tf_kv_pool *pool, const tf_streams *streams,
                   const void *k_rows, const void *v_rows, int32_t rows,
                   void *stream);

/* The state copy (TensorFold #1620, opening comment, "Kept states" bullet:
 * a kept state is copied by walking the slot's pages).  For every stream s
 * and position j < src->lens[s], the head_dim bf16 values of K and of V of
 * every KV head are copied bit for bit from src_pool page
 * src->table[s][j / src page_size], slot j % src page_size, to dst_pool page
 * dst_table[s][j / dst page_size], slot j % dst page_size.  Nothing else of
 * dst_pool is written.  The pools may be the same or differ in n_pages and
 * page_size; n_kv_heads and head_dim must match.  A linear buffer is a pool
 * with one page per stream (page_size >= the state's length), so keeping a
 * state (pages to linear), resuming it (linear to pages) and moving it
 * between pages are all this call.
 *  src, src_pool  as for the attention calls (src->max_len bounds every
 *                 lens[s] and sizes the launch)
 *  dst_table      device int32 [n_streams][dst_table_stride], caller-owned;
 *                 dst_table_stride * dst page_size must be >= src->max_len
 *  status         optional device uint32 (4-byte aligned): TF_DEV_BAD_LEN and
 *                 TF_DEV_BAD_PAGE are ORed in for skipped streams and pieces
 * The copied source and destination ranges must not overlap.  Returns
 * TF_OK, TF_EINVAL (bad or mismatched arguments), TF_EUNSUPPORTED (head_dim)
 * or TF_ECUDA; enqueued on `stream`. */
TF_API int tf_kv_copy_state(const tf_kv_pool *src_pool, const tf_streams *src,
                            const tf_kv_pool *dst_pool, const int32_t *dst_table,
                            int32_t dst_table_stride, uint32_t *status, void *stream);

/* Workspace bytes an attention call with these arguments needs on the
 * current device (0 on a bad argument).  Follows the scratch convention of
 * the metrale page "metrale_model_arch/glm5next_dsa/select.rs": scratch is
 * owned by the caller, sized once from the largest shape it will run and
 * reused across steps (the DsaSelectScratch doc comment), and a call whose
 * plan needs more than was given fails before any launch instead of
 * overrunning it (DsaSelectScratch::fits; here TF_ENOSPACE).  The figure is
 * for any of the attention calls
 * with these arguments (tf_paged_attn_verify_tree included).  The workspace holds split-context
 * partial results and, in its first 4 bytes, the device status word, which
 * the calls only OR bits into: zero those 4 bytes once after allocating
 * (cudaMemset, or one tf_workspace_status call).  The rest needs no
 * initialisation.  One workspace may serve later calls on the same stream;
 * calls that may run concurrently need separate workspaces. */
TF_API size_t tf_paged_attn_workspace_bytes(const tf_kv_pool *pool,
                                     const tf_streams *streams,
                                     int32_t n_q_heads, int32_t rows);

/* Single-row decode (TensorFold #1620, opening comment, "Reads": decode).
 * Same as tf_paged_attn_verify with rows = 1. */
TF_API int tf_paged_attn_decode(const tf_kv_pool *pool, const tf_streams *streams,
                         const void *q, int32_t n_q_heads, float scale,
                         float *out, void *workspace, size_t workspace_bytes,
                         void *stream);

/* Draft-verify window (TensorFold #1620 "Reads": drafted verify; TensorFold
 * #2730 "What this changes": the pending token plus up to seven drafts).
 * rows in [1, 8]; row r sees positions 0 .. lens[s] - rows + r. */
TF_API int tf_paged_attn_verify(const tf_kv_pool *pool, const tf_streams *streams,
                         const void *q, int32_t n_q_heads, int32_t rows,
                         float scale, float *out, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Draft-verify window whose rows form a draft tree (TensorFold #1620,
 * opening comment, first and Reads bullets: drafted verify runs through
 * "tree attention" kernels whose key groups are the 512-position pages; the
 * pages give no mask, so this reading: a window of `rows` drafted tokens,
 * laid out in order, each seeing the positions before the window and the
 * window rows named by its mask).
 *  tree_masks  device, uint8 [n_streams][rows], caller-owned, read during the
 *              call: bit c of tree_masks[s][r] set means row r of stream s
 *              sees window row c (position lens[s] - rows + c).  A draft tree
 *              gives row r its ancestors and itself; the causal window of
 *              tf_paged_attn_verify is the chain mask 2^(r+1) - 1.  Bits at or
 *              above `rows` are ignored.  A row that sees no position at all
 *              (no context before the window and an empty mask) gets NaN.
 * Everything else (arguments, layouts, results, the workspace, errors) is
 * as tf_paged_attn_verify; TF_EINVAL also when tree_masks is null (with
 * n_streams > 0).  Head dim 128
 * calls with more than 64 query rows per KV head (G * rows) read each K/V
 * tile once per 64 rows. */
TF_API int tf_paged_attn_verify_tree(const tf_kv_pool *pool, const tf_streams *streams,
                              const void *q, int32_t n_q_heads, int32_t rows,
                              const uint8_t *tree_masks, float scale, float *out,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Chunked prompt rows (TensorFold #1620 "Reads": prompts through the paged
 * prompt kernels).  The same causal rule as verify for a chunk of
 * rows in [1, 4096] positions: the chunk is the last `rows` positions. */
TF_API int tf_paged_attn_prompt(const tf_kv_pool *pool, const tf_streams *streams,
                         const void *q, int32_t n_q_heads, int32_t rows,
                         float scale, float *out, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Single-row decode that allocates nothing and takes no workspace.  The
 * source pages have no counterpart of this call.
 * For callers that cannot allocate device memory for a workspace: a
 * plug-in hosted by an engine that hands it only its input and output
 * buffers, or a serving loop that must not call cudaMalloc once running.
 * The split-context scratch is one static device array of 8 MiB inside
 * this library, held by every GPU that loads it until the process exits.
 * Arguments, results and errors are those of tf_paged_attn_decode, except:
 *  - TF_ENOSPACE when the call would need more than the 8 MiB of scratch
 *    (tf_paged_attn_workspace_bytes with rows = 1 gives the need);
 *  - the first call on each device looks the array's device address up
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture on the device;
 *  - every call on a device shares the one array, which keeps the last
 *    call's contents: calls whose kernels may overlap on the GPU (other
 *    streams, other host threads) race and must be serialised by the caller;
 *  - device-side status bits are not reported (streams with a bad length
 *    still get NaN outputs); use tf_paged_attn_decode to read them. */
TF_API int tf_paged_attn_decode_noalloc(const tf_kv_pool *pool,
                                        const tf_streams *streams,
                                        const void *q, int32_t n_q_heads,
                                        float scale, float *out, void *stream);

/* Reads the workspace's device status word (TF_DEV_* bits accumulated by
 * the attention calls since the last read) into *flags and clears it.
 * Synchronises `stream`.  Returns TF_OK, TF_EINVAL or TF_ECUDA.
 * The source pages have no counterpart of this call: their launchers check
 * host arguments only (the select.rs page's plan and fits), while lens and
 * table here are device data that only the kernels can check. */
TF_API int tf_workspace_status(void *workspace, uint32_t *flags, void *stream);

/* A static, human-readable name for a status code.  The select.rs page's
 * plan and fits refuse a bad shape or a short scratch with a message that
 * names what was wrong; a C caller gets the code from the call and its name
 * from here. */
TF_API const char *tf_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* TF_PAGED_H */
