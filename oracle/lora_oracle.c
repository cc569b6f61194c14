/*
 * lora_oracle.c -- the CPU oracle for the multi-LoRA delta path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, obviously correct
 * restatement of what the path computes, in fp64 with one loop per row.  Only
 * the test suite, the package smoke check and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header or table with the CUDA library and
 * includes nothing from it; the library never loads it.
 *
 * Sources (web pages on multi-LoRA serving):
 *  - "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU", section "Why can't
 *    you just merge LoRA weights into the base model?": y = xW + (x A_i) B_i *
 *    (alpha / r); the xW term is shared, the delta is per request.
 *  - same page, section "How much memory does one LoRA adapter actually cost?":
 *    for a d_out x d_in matrix a rank-r adapter stores A: r x d_in and
 *    B: d_out x r, so r * (d_in + d_out) parameters.
 *  - "Serving Many LoRA Adapters From One Base Model", section "How it works":
 *    the column form W.x + (B.A).x, and "Batching across adapters": each row
 *    of a mixed batch gets its own adapter's correction.
 *  - same page, worked example: adapter=None is the plain base (no delta).
 *  - "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU", section "How does
 *    one batch run 30 different adapters at once?": the batch carries an index
 *    vector mapping each row to an adapter id; grouping rows by adapter is the
 *    segmented gather.
 *  - "Multi-LoRA Serving: Sharing One GPU Across Adapters", section "How S-LoRA
 *    Proved the Model": adapter weights live in a paged pool.
 *
 * Readings of points the pages leave open:
 *  - With A stored r x d_in and B stored d_out x r, the row form's product
 *    (x A_i) contracts x with each row of A_i, i.e. v = A_i x (column form),
 *    then delta = B_i v.  Both pages' forms are this one computation.
 *  - r in alpha / r is the adapter's own (true) rank.
 *  - Id -1 means "no adapter": the row keeps its base output unchanged.  An
 *    adapter whose rank on this matrix is 0 also leaves the row unchanged.
 *  - An id outside [-1, n_slots) or naming a slot with no weights is invalid:
 *    the row is left unchanged and counted.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------- */
/* Per-row LoRA delta, fp64.                                               */
/* ---------------------------------------------------------------------- */

typedef struct {
    int t_begin, t_end;
    int d_in, d_out;
    const double *x;          /* [T][d_in]  */
    const double *y_in;       /* [T][d_out] */
    const int32_t *ids;       /* [T]        */
    int n_slots;
    const double *const *A;   /* per slot: [rank][d_in] or NULL */
    const double *const *B;   /* per slot: [d_out][rank] or NULL */
    const int32_t *rank;      /* per slot */
    const double *alpha;      /* per slot */
    double *y_out;            /* [T][d_out] */
    double *v_out;            /* optional [T][ldv] */
    int ldv;
    int32_t bad;              /* rows with an invalid id */
} apply_job;

/* Classify row t: returns the slot whose delta applies, or -1 for "row
 * unchanged".  Sets *bad when the id is invalid. */
static int row_slot(const apply_job *j, int t, int *bad)
{
    int a = j->ids[t];
    *bad = 0;
    if (a == -1) return -1;                       /* adapter=None */
    if (a < -1 || a >= j->n_slots) { *bad = 1; return -1; }
    if (j->rank[a] <= 0) return -1;               /* not adapted here */
    if (j->A[a] == NULL || j->B[a] == NULL) { *bad = 1; return -1; }
    return a;
}

static void *apply_rows(void *arg)
{
    apply_job *j = (apply_job *)arg;
    for (int t = j->t_begin; t < j->t_end; ++t) {
        const double *xt = j->x + (size_t)t * j->d_in;
        const double *yt = j->y_in + (size_t)t * j->d_out;
        double *ot = j->y_out + (size_t)t * j->d_out;
        int bad;
        int a = row_slot(j, t, &bad);
        j->bad += bad;
        if (a < 0) {
            for (int n = 0; n < j->d_out; ++n) ot[n] = yt[n];
            continue;
        }
        int r = j->rank[a];
        const double *A = j->A[a];
        const double *B = j->B[a];
        double s = j->alpha[a] / (double)r;       /* alpha / r */

        /* v = A x : one dot product per adapter row */
        double *v = (double *)malloc(sizeof(double) * (size_t)r);
        for (int q = 0; q < r; ++q) {
            double acc = 0.0;
            for (int k = 0; k < j->d_in; ++k)
                acc += xt[k] * A[(size_t)q * j->d_in + k];
            v[q] = acc;
        }
        if (j->v_out) {
            double *vt = j->v_out + (size_t)t * j->ldv;
            for (int q = 0; q < j->ldv; ++q) vt[q] = (q < r) ? v[q] : 0.0;
        }
        /* y = y_in + s * (B v) */
        for (int n = 0; n < j->d_out; ++n) {
            double acc = 0.0;
            for (int q = 0; q < r; ++q)
                acc += B[(size_t)n * r + q] * v[q];
            ot[n] = yt[n] + s * acc;
        }
        free(v);
    }
    return NULL;
}

/*
 * y_out[t] = y_in[t] + (alpha_a / r_a) * B_a (A_a x[t])   with a = ids[t],
 * or y_out[t] = y_in[t] when the row has no (valid) adapter.
 *
 * x, y_in, y_out are dense row-major fp64 arrays.  A[a] is r_a x d_in and
 * B[a] is d_out x r_a, both dense row-major fp64 (the adapter's own rank, no
 * padding).  v_out (optional, may be NULL) receives v = A_a x[t] for each
 * adapted row, zero-filled up to ldv; rows left unchanged are not written.
 * Rows are split into contiguous ranges over n_threads threads; each row's
 * arithmetic is the same whatever the thread count.  Returns the number of
 * rows whose id was invalid.
 */
int oracle_lora_apply(int T, int d_in, int d_out,
                      const double *x, const double *y_in, const int32_t *ids,
                      int n_slots, const double *const *A,
                      const double *const *B, const int32_t *rank,
                      const double *alpha, double *y_out,
                      double *v_out, int ldv, int n_threads)
{
    if (T <= 0) return 0;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > T) n_threads = T;
    apply_job *jobs = (apply_job *)calloc((size_t)n_threads, sizeof(apply_job));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    for (int i = 0; i < n_threads; ++i) {
        apply_job *j = &jobs[i];
        j->t_begin = (int)((long long)T * i / n_threads);
        j->t_end = (int)((long long)T * (i + 1) / n_threads);
        j->d_in = d_in; j->d_out = d_out;
        j->x = x; j->y_in = y_in; j->ids = ids; j->n_slots = n_slots;
        j->A = A; j->B = B; j->rank = rank; j->alpha = alpha;
        j->y_out = y_out; j->v_out = v_out; j->ldv = ldv; j->bad = 0;
    }
    for (int i = 1; i < n_threads; ++i) pthread_create(&th[i], NULL, apply_rows, &jobs[i]);
    apply_rows(&jobs[0]);
    for (int i = 1; i < n_threads; ++i) pthread_join(th[i], NULL);
    int bad = 0;
    for (int i = 0; i < n_threads; ++i) bad += jobs[i].bad;
    free(jobs); free(th);
    return bad;
}

/* ---------------------------------------------------------------------- */
/* The shared base term, fp64.                                             */
/* ---------------------------------------------------------------------- */

typedef struct {
    int t_begin, t_end, d_in, d_out;
    const double *x;   /* [T][d_in] */
    const double *W;   /* [d_out][d_in] */
    double *out;       /* [T][d_out] */
} linear_job;

static void *linear_rows(void *arg)
{
    linear_job *j = (linear_job *)arg;
    for (int t = j->t_begin; t < j->t_end; ++t) {
        const double *xt = j->x + (size_t)t * j->d_in;
        for (int n = 0; n < j->d_out; ++n) {
            const double *wn = j->W + (size_t)n * j->d_in;
            double acc = 0.0;
            for (int k = 0; k < j->d_in; ++k) acc += xt[k] * wn[k];
            j->out[(size_t)t * j->d_out + n] = acc;
        }
    }
    return NULL;
}

/*
 * out[t][n] = sum_k x[t][k] * W[n][k]: the base term xW that every row shares
 * ("Multi-LoRA Serving: Why 100 Adapters Fit on One GPU", section "Why can't
 * you just merge LoRA weights into the base model?").  W is stored as the
 * d_out x d_in matrix of the column form W.x ("Serving Many LoRA Adapters
 * From One Base Model", section "How it works"), so the row form's xW is the
 * product of x with the transpose of this W.  Rows are split over n_threads
 * threads; each output is one k-ascending dot product whatever the count.
 */
void oracle_linear(int T, int d_in, int d_out, const double *x,
                   const double *W, double *out, int n_threads)
{
    if (T <= 0) return;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > T) n_threads = T;
    linear_job *jobs = (linear_job *)calloc((size_t)n_threads, sizeof(linear_job));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    for (int i = 0; i < n_threads; ++i) {
        linear_job *j = &jobs[i];
        j->t_begin = (int)((long long)T * i / n_threads);
        j->t_end = (int)((long long)T * (i + 1) / n_threads);
        j->d_in = d_in; j->d_out = d_out; j->x = x; j->W = W; j->out = out;
    }
    for (int i = 1; i < n_threads; ++i) pthread_create(&th[i], NULL, linear_rows, &jobs[i]);
    linear_rows(&jobs[0]);
    for (int i = 1; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(jobs); free(th);
}

/*
 * Expand step alone: y_out[t] = y_in[t] + (alpha_a / r_a) * B_a v[t], with the
 * caller's v[t] (first r_a entries of row t of a [T][ldv] array).  Same row
 * rules as oracle_lora_apply.  Returns the number of invalid ids.
 */
int oracle_lora_expand(int T, int d_out, const double *v, int ldv,
                       const double *y_in, const int32_t *ids, int n_slots,
                       const double *const *B, const int32_t *rank,
                       const double *alpha, double *y_out)
{
    int bad_total = 0;
    for (int t = 0; t < T; ++t) {
        const double *yt = y_in + (size_t)t * d_out;
        double *ot = y_out + (size_t)t * d_out;
        int a = ids[t];
        int ok = 1;
        if (a == -1) ok = 0;
        else if (a < -1 || a >= n_slots) { ok = 0; ++bad_total; }
        else if (rank[a] <= 0) ok = 0;
        else if (B[a] == NULL) { ok = 0; ++bad_total; }
        if (!ok) {
            for (int n = 0; n < d_out; ++n) ot[n] = yt[n];
            continue;
        }
        int r = rank[a];
        double s = alpha[a] / (double)r;
        const double *vt = v + (size_t)t * ldv;
        for (int n = 0; n < d_out; ++n) {
            double acc = 0.0;
            for (int q = 0; q < r; ++q) acc += B[a][(size_t)n * r + q] * vt[q];
            ot[n] = yt[n] + s * acc;
        }
    }
    return bad_total;
}

/* ---------------------------------------------------------------------- */
/* Index vector -> segments (stable grouping of rows by adapter id).       */
/* ---------------------------------------------------------------------- */

/*
 * Group the rows of a batch by adapter id, the segmented layout a gather
 * kernel walks: segments in ascending slot order, and inside a segment the
 * rows in ascending row order (a stable grouping).  Rows with id -1 or an
 * invalid id belong to no segment.  valid[s] (may be NULL) marks the slots
 * that can be used; a row naming a slot with valid[s] == 0 is invalid.
 *
 * Outputs: perm[0..n_active) row indices; seg_start[0..n_segs] offsets into
 * perm; seg_slot[0..n_segs) the slot of each segment.  Returns n_segs, and
 * writes the number of rows with invalid ids to *n_bad.
 */
int oracle_group_rows(int T, const int32_t *ids, int n_slots,
                      const uint8_t *valid, int32_t *perm, int32_t *seg_start,
                      int32_t *seg_slot, int32_t *n_active, int32_t *n_bad)
{
    int n = 0, s = 0, bad = 0;
    for (int t = 0; t < T; ++t) {
        int a = ids[t];
        if (a == -1) continue;
        if (a < -1 || a >= n_slots || (valid && !valid[a])) ++bad;
    }
    for (int slot = 0; slot < n_slots; ++slot) {
        if (valid && !valid[slot]) continue;
        int first = 1;
        for (int t = 0; t < T; ++t) {
            if (ids[t] != slot) continue;
            if (first) { seg_start[s] = n; seg_slot[s] = slot; ++s; first = 0; }
            perm[n++] = t;
        }
    }
    seg_start[s] = n;
    *n_active = n;
    *n_bad = bad;
    return s;
}

/* ---------------------------------------------------------------------- */
/* Paged adapter pool: logical -> physical address.                       */
/* ---------------------------------------------------------------------- */

/*
 * A slot's weights occupy a logical byte range [0, slot_bytes) cut into pages
 * of page_bytes; page_table[slot * pages_per_slot + p] names the physical page
 * holding logical page p.  Physical byte = physical page * page_bytes +
 * offset inside the page.  (Unified paging of adapter weights.)
 */
long long oracle_pool_locate(int slot, long long logical_off,
                             const int32_t *page_table, int pages_per_slot,
                             long long page_bytes)
{
    long long p = logical_off / page_bytes;
    long long inside = logical_off % page_bytes;
    long long phys_page = page_table[(long long)slot * pages_per_slot + p];
    return phys_page * page_bytes + inside;
}

/*
 * Byte layout of one slot, as the library's public header documents it: the
 * targets follow one another in order; target t holds A (r_max rows of d_in
 * bf16, row j = adapter row j) and then B transposed (r_max rows of d_out
 * bf16, row j = column j of B); each of these two blocks starts on a
 * 256-byte boundary.  Writes a_off[t], bt_off[t] and returns slot_bytes.
 */
long long oracle_slot_layout(int n_targets, const int32_t *d_in,
                             const int32_t *d_out, int r_max,
                             long long *a_off, long long *bt_off)
{
    long long off = 0;
    for (int t = 0; t < n_targets; ++t) {
        long long a_bytes = (long long)r_max * d_in[t] * 2;
        long long b_bytes = (long long)r_max * d_out[t] * 2;
        a_off[t] = off;
        off += (a_bytes + 255) / 256 * 256;
        bt_off[t] = off;
        off += (b_bytes + 255) / 256 * 256;
    }
    return off;
}

/* ---------------------------------------------------------------------- */
/* Adapter sizing.                                                          */
/* ---------------------------------------------------------------------- */

/*
 * Parameter count of a rank-r adapter.  An adapted matrix W of shape
 * d_out x d_in gets A (r x d_in) and B (d_out x r): r d_in + d_out r
 * parameters.  A layer adapts n_targets matrices (shapes d_in[t] x d_out[t]);
 * the adapter covers n_layers such layers.
 */
long long oracle_lora_params(int n_targets, const long long *d_in, const long long *d_out,
                             long long n_layers, long long rank)
{
    long long per_layer = 0;
    for (int t = 0; t < n_targets; ++t) {
        long long a_params = rank * d_in[t];   /* A */
        long long b_params = d_out[t] * rank;  /* B */
        per_layer += a_params + b_params;
    }
    return per_layer * n_layers;
}
