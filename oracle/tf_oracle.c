/*
 * tf_oracle.c -- plain fp64 CPU oracle for attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library,
 * its binding) may include, link or call this file.  Only tests/, the smoke
 * check and the benchmark's CPU-baseline leg use it.
 *
 * It shares no code, header or constant with the GPU path.  It works on
 * LINEAR (unpaged) caches: stream s keeps its keys and values as
 * [len_s][n_kv_heads][head_dim] bf16 rows, position-major.  Paging is a
 * storage detail of the GPU path; the oracle never sees a page.
 *
 * What it computes (sources):
 *  - TensorFold pull request #1620 ("Kolibri-1's full layers take their K/V
 *    from pages of the core pool"), opening comment, the Writes / Reads
 *    bullets: new K/V rows are copied into the stream's pages (the row
 *    write), and decode, drafted verify and prompt rows attend over the keys
 *    the stream holds.  Its kernel-contract bullet checks paged results
 *    against linear caches; its "kolibri-pages" bullet states linear and
 *    paged give byte-equal logits.
 *  - TensorFold pull request #2730 ("an eight-row verify window"), section
 *    "What this changes": a verify window is the pending token plus up to
 *    seven drafts; its checklist requires drafted output to equal undrafted
 *    output, so row r of a window sees exactly the keys that a plain decode
 *    at that position would see: causal inside the window.
 *
 * The pages print no formula; this is the textbook definition of softmax
 * attention with grouped-query heads, written out directly:
 *
 *   for stream s, window row r (0 <= r < W), query head h (0 <= h < Hq):
 *     kh = h / G                      (contiguous query-head groups)
 *     t  = len_s - W + r              (position of row r; it sees 0..t)
 *     x_j = scale * sum_i q[s][r][h][i] * K_s[j][kh][i]      j = 0..t
 *     o[s][r][h][i] = sum_j exp(x_j - max x) V_s[j][kh][i] / sum_j exp(x_j - max x)
 *
 * Tree-mask verify (tfo_attend_units_tree).  The same page names the
 * verify kernels "tree attention" and calls the 512-position pages its key
 * groups (opening comment, first bullet and Reads bullet); it gives no mask.
 * The reading used here: a window of W rows is a draft tree laid out in
 * order, and row r carries a bitmask tree[s][r] over the window's rows --
 * bit c set means row r sees window row c (its ancestors and itself).  Every
 * position before the window is seen by every row.  So row r attends to
 *     { j < len_s - W }  U  { len_s - W + c : bit c of tree[s][r] }
 * and the causal window above is the chain mask tree[s][r] = 2^(r+1) - 1.
 * A row whose set is empty is refused (status -1).
 *
 * Everything is fp64; bf16 inputs are exact in fp64.  One unit (s, r, h)
 * is computed by one thread start to finish in a fixed order, so the result
 * does not depend on how many threads run.
 *
 * The row write (tfo_put_rows) is the plain host scatter: row r of stream s
 * goes to page table[s][pos / P], slot pos % P, with pos = len_s - W + r.
 *
 * The state copy (tfo_copy_state) follows the same page's "Kept states"
 * bullet (opening comment): a kept state is copied by walking the slot's
 * pages.  Reading: for every stream s, position j < len_s and KV head kh,
 * the d values of K (and of V) at src page src_table[s][j / Ps], slot
 * j % Ps are copied to dst page dst_table[s][j / Pd], slot j % Pd.  A
 * linear buffer is a pool whose one page per stream holds the whole state,
 * so keeping (pages to linear), resuming (linear to pages) and reusing
 * pages (pages to pages) are the one copy.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is the high half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const uint16_t *q;      /* [S][W][Hq][d] */
    const uint16_t *k;      /* stream s at k + kv_off[s]: [len_s][Hkv][d] */
    const uint16_t *v;
    const int64_t *kv_off;
    const int32_t *lens;
    int32_t S, W, Hkv, G, d;
    double scale;
    const uint8_t *tree;    /* NULL (causal), or [S][W] row masks */
    const int32_t *units;   /* n_units triples (s, r, h) */
    int64_t n_units;
    double *out;            /* [n_units][d] */
    int32_t nthreads;
    int32_t tid;
    int32_t status;
} attend_job;

/* Whether row r of stream s sees position j (the definitions above). */
static int row_sees(const attend_job *J, int32_t s, int32_t r, int64_t j)
{
    const int64_t base = (int64_t)J->lens[s] - J->W;  /* the window's first position */
    if (j < base)
        return 1;
    if (j >= J->lens[s])
        return 0;
    if (J->tree == NULL)
        return j <= base + r;
    return (J->tree[(int64_t)s * J->W + r] >> (j - base)) & 1;
}

/* One output row, straight from the definition above: the scores of the
 * positions the row sees, in position order, then the softmax and the
 * weighted sum of their values. */
static int attend_one(const attend_job *J, int32_t s, int32_t r, int32_t h,
                      double *o, double *x, double *w, int64_t *pos)
{
    const int32_t Hq = J->Hkv * J->G;
    const int32_t d = J->d;
    const int32_t kh = h / J->G;
    const uint16_t *qrow = J->q + (((int64_t)s * J->W + r) * Hq + h) * d;
    const uint16_t *ks = J->k + J->kv_off[s];
    const uint16_t *vs = J->v + J->kv_off[s];
    int64_t j, n = 0;
    int32_t i;
    double mx, l;

    if ((int64_t)J->lens[s] - J->W + r < 0)
        return -1;
    for (j = 0; j < J->lens[s]; ++j)
        if (row_sees(J, s, r, j))
            pos[n++] = j;
    if (n == 0)
        return -1;
    for (j = 0; j < n; ++j) {
        const uint16_t *krow = ks + (pos[j] * J->Hkv + kh) * d;
        double acc = 0.0;
        for (i = 0; i < d; ++i)
            acc += bf16_to_double(qrow[i]) * bf16_to_double(krow[i]);
        x[j] = J->scale * acc;
    }
    mx = x[0];
    for (j = 1; j < n; ++j)
        if (x[j] > mx)
            mx = x[j];
    l = 0.0;
    for (j = 0; j < n; ++j) {
        w[j] = exp(x[j] - mx);
        l += w[j];
    }
    for (i = 0; i < d; ++i)
        o[i] = 0.0;
    for (j = 0; j < n; ++j) {
        const uint16_t *vrow = vs + (pos[j] * J->Hkv + kh) * d;
        for (i = 0; i < d; ++i)
            o[i] += w[j] * bf16_to_double(vrow[i]);
    }
    for (i = 0; i < d; ++i)
        o[i] /= l;
    return 0;
}

static void *attend_worker(void *arg)
{
    attend_job *J = (attend_job *)arg;
    int64_t maxlen = 1, u;
    int32_t s;
    double *x, *w;
    int64_t *pos;

    for (s = 0; s < J->S; ++s)
        if (J->lens[s] > maxlen)
            maxlen = J->lens[s];
    x = (double *)malloc(sizeof(double) * (size_t)maxlen);
    w = (double *)malloc(sizeof(double) * (size_t)maxlen);
    pos = (int64_t *)malloc(sizeof(int64_t) * (size_t)maxlen);
    if (!x || !w || !pos) {
        J->status = -2;
        free(x);
        free(w);
        free(pos);
        return NULL;
    }
    for (u = J->tid; u < J->n_units; u += J->nthreads) {
        const int32_t *t3 = J->units + 3 * u;
        if (attend_one(J, t3[0], t3[1], t3[2], J->out + u * J->d, x, w, pos) != 0) {
            J->status = -1;
            break;
        }
    }
    free(x);
    free(w);
    free(pos);
    return NULL;
}

/*
 * Attention for a list of (stream, window row, query head) units, with the
 * window's rows either causal (tree == NULL) or under per-row tree masks.
 * Returns 0, or -1 on a bad argument (a row before position 0, a unit out
 * of range, a row that sees nothing), -2 when memory runs out.
 */
int tfo_attend_units_tree(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int64_t *kv_off, const int32_t *lens, int32_t S,
                          int32_t W, int32_t Hkv, int32_t G, int32_t d, double scale,
                          const uint8_t *tree, const int32_t *units, int64_t n_units,
                          double *out, int32_t nthreads)
{
    attend_job *jobs;
    pthread_t *th;
    int64_t u;
    int32_t t, st = 0;

    if (S <= 0 || W <= 0 || Hkv <= 0 || G <= 0 || d <= 0 || n_units < 0)
        return -1;
    if (tree != NULL && W > 8)
        return -1;  /* one mask byte per row */
    for (u = 0; u < n_units; ++u) {
        const int32_t *t3 = units + 3 * u;
        if (t3[0] < 0 || t3[0] >= S || t3[1] < 0 || t3[1] >= W || t3[2] < 0 ||
            t3[2] >= Hkv * G || lens[t3[0]] < W)
            return -1;
    }
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    jobs = (attend_job *)calloc((size_t)nthreads, sizeof *jobs);
    th = (pthread_t *)calloc((size_t)nthreads, sizeof *th);
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return -2;
    }
    for (t = 0; t < nthreads; ++t) {
        attend_job *J = &jobs[t];
        J->q = q; J->k = k; J->v = v; J->kv_off = kv_off; J->lens = lens;
        J->S = S; J->W = W; J->Hkv = Hkv; J->G = G; J->d = d; J->scale = scale;
        J->tree = tree; J->units = units; J->n_units = n_units; J->out = out;
        J->nthreads = nthreads; J->tid = t; J->status = 0;
    }
    if (nthreads == 1) {
        attend_worker(&jobs[0]);
    } else {
        for (t = 0; t < nthreads; ++t)
            if (pthread_create(&th[t], NULL, attend_worker, &jobs[t]) != 0) {
                /* fall back to running it on this thread */
                attend_worker(&jobs[t]);
                th[t] = 0;
            }
        for (t = 0; t < nthreads; ++t)
            if (th[t])
                pthread_join(th[t], NULL);
    }
    for (t = 0; t < nthreads; ++t)
        if (jobs[t].status != 0)
            st = jobs[t].status;
    free(jobs);
    free(th);
    return st;
}

/* The causal window: tfo_attend_units_tree without masks. */
int tfo_attend_units(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int64_t *kv_off, const int32_t *lens, int32_t S,
                     int32_t W, int32_t Hkv, int32_t G, int32_t d, double scale,
                     const int32_t *units, int64_t n_units, double *out,
                     int32_t nthreads)
{
    return tfo_attend_units_tree(q, k, v, kv_off, lens, S, W, Hkv, G, d, scale, NULL, units,
                                 n_units, out, nthreads);
}

/*
 * The row write: copy `W` new rows per stream into their pages.
 * Pools are [n_pages][Hkv][P][d] bf16; table is [S][table_stride] int32;
 * rows are [S][W][Hkv][d].  Bytes are copied, never converted.
 * Returns 0, or -1 when a position or page id falls outside its range.
 */
int tfo_put_rows(uint16_t *k_pool, uint16_t *v_pool, int32_t n_pages,
                 int32_t Hkv, int32_t P, int32_t d, const int32_t *table,
                 int32_t table_stride, const int32_t *lens, int32_t S,
                 const uint16_t *k_rows, const uint16_t *v_rows, int32_t W)
{
    int32_t s, r, kh;
    for (s = 0; s < S; ++s) {
        if (lens[s] < W || lens[s] > (int64_t)table_stride * P)
            return -1;
        for (r = 0; r < W; ++r) {
            const int64_t pos = (int64_t)lens[s] - W + r;
            const int32_t page = table[(int64_t)s * table_stride + pos / P];
            const int64_t slot = pos % P;
            if (page < 0 || page >= n_pages)
                return -1;
            for (kh = 0; kh < Hkv; ++kh) {
                const int64_t dst = (((int64_t)page * Hkv + kh) * P + slot) * d;
                const int64_t src = (((int64_t)s * W + r) * Hkv + kh) * d;
                memcpy(k_pool + dst, k_rows + src, sizeof(uint16_t) * (size_t)d);
                memcpy(v_pool + dst, v_rows + src, sizeof(uint16_t) * (size_t)d);
            }
        }
    }
    return 0;
}

/*
 * The state copy: positions [0, lens[s]) of every KV head of every stream,
 * from the source pool's pages to the destination pool's pages, each found
 * through its own table.  Pools are [n_pages][Hkv][P][d] bf16 (the two may
 * differ in n_pages and P).  Bytes are copied, never converted.
 * Returns 0, or -1 when a position or page id falls outside its range.
 */
int tfo_copy_state(const uint16_t *src_k, const uint16_t *src_v, int32_t src_n_pages,
                   int32_t src_P, const int32_t *src_table, int32_t src_stride,
                   uint16_t *dst_k, uint16_t *dst_v, int32_t dst_n_pages, int32_t dst_P,
                   const int32_t *dst_table, int32_t dst_stride, int32_t Hkv, int32_t d,
                   const int32_t *lens, int32_t S)
{
    int32_t s, kh;
    int64_t j;
    for (s = 0; s < S; ++s) {
        if (lens[s] < 0 || lens[s] > (int64_t)src_stride * src_P ||
            lens[s] > (int64_t)dst_stride * dst_P)
            return -1;
        for (j = 0; j < lens[s]; ++j) {
            const int32_t sp = src_table[(int64_t)s * src_stride + j / src_P];
            const int32_t dp = dst_table[(int64_t)s * dst_stride + j / dst_P];
            if (sp < 0 || sp >= src_n_pages || dp < 0 || dp >= dst_n_pages)
                return -1;
            for (kh = 0; kh < Hkv; ++kh) {
                const int64_t from = (((int64_t)sp * Hkv + kh) * src_P + j % src_P) * d;
                const int64_t to = (((int64_t)dp * Hkv + kh) * dst_P + j % dst_P) * d;
                memcpy(dst_k + to, src_k + from, sizeof(uint16_t) * (size_t)d);
                memcpy(dst_v + to, src_v + from, sizeof(uint16_t) * (size_t)d);
            }
        }
    }
    return 0;
}
