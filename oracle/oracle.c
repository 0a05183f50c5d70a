/*
 * oracle.c -- plain fp64 CPU reference of Re-ttention's attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the bench's CPU
 * baseline / reference arm use it.  It shares no code with the CUDA library.
 *
 * What it follows (Re-ttention: Ultra Sparse Visual Generation via Attention
 * Statistical Reshape, project page):
 *   - teaser: sparse attention is corrected with statistics kept from an
 *     earlier denoising step, so that it recovers the full attention
 *     distribution;
 *   - Abstract: the sparse step sees a small part of the tokens, and the
 *     reshape undoes the shift that normalising over that subset causes,
 *     using the softmax statistics of an earlier step;
 *   - mechanism highlight: the full/sparse softmax-denominator ratio is reused
 *     and the residual contribution of masked-out tokens is cached.
 * The pages give no formula, mask rule or precision.  The readings taken here
 * (block mean pooling, top-k with forced prefix blocks and lower-index
 * tie-break, the reshape o = (N' + e^{m_c-m'} U) / (Z' * Z_full / Z_kept))
 * are listed with their reasons in the repository's design notes.
 *
 * Every floating-point step is fp64, every reduction runs in natural index
 * order, nothing is blocked, fused or reordered.  Inputs are bf16 bit
 * patterns widened exactly to fp64.  Parallelism is over independent rows
 * only (pthreads), which does not change any result.
 *
 * Parity status of each function is stated above it.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Exact bf16 -> fp64 widening: a bf16 value is the top half of an fp32. */
static double bf16_to_f64(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int64_t n_blocks_of(int64_t n, int64_t bs) { return (n + bs - 1) / bs; }

/* ------------------------------------------------------------------------ */
/* Block pooling (pinned: numpy mean over the block's real tokens).          */
/* out[bh][b][c] = mean over tokens i of block b (i < n) of x[bh][i][c],     */
/* for logical columns c < d.  The last block of a ragged sequence is        */
/* averaged over its real tokens only.                                       */
/* ------------------------------------------------------------------------ */
int orc_pool_blocks(const uint16_t *x, int64_t bh_count, int64_t n, int64_t dpad,
                    int64_t d, int64_t bs, double *out) {
    if (!x || !out || bh_count < 0 || n <= 0 || d <= 0 || dpad < d || bs <= 0) return 1;
    int64_t nb = n_blocks_of(n, bs);
    for (int64_t bh = 0; bh < bh_count; ++bh) {
        for (int64_t b = 0; b < nb; ++b) {
            int64_t i0 = b * bs, i1 = i0 + bs < n ? i0 + bs : n;
            double *o = out + (bh * nb + b) * d;
            for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t i = i0; i < i1; ++i) {
                const uint16_t *row = x + (bh * n + i) * dpad;
                for (int64_t c = 0; c < d; ++c) o[c] += bf16_to_f64(row[c]);
            }
            for (int64_t c = 0; c < d; ++c) o[c] /= (double)(i1 - i0);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block scores (pinned: numpy matmul of the pooled means).                  */
/* s[bh][qb][kb] = scale * sum_c pq[bh][qb][c] * pk[bh][kb][c].              */
/* ------------------------------------------------------------------------ */
int orc_block_scores(const double *pq, const double *pk, int64_t bh_count, int64_t nb,
                     int64_t d, double scale, double *s) {
    if (!pq || !pk || !s || bh_count < 0 || nb <= 0 || d <= 0) return 1;
    for (int64_t bh = 0; bh < bh_count; ++bh)
        for (int64_t qb = 0; qb < nb; ++qb)
            for (int64_t kb = 0; kb < nb; ++kb) {
                const double *a = pq + (bh * nb + qb) * d, *b = pk + (bh * nb + kb) * d;
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) acc += a[c] * b[c];
                s[(bh * nb + qb) * nb + kb] = scale * acc;
            }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Kept-block selection (pinned: brute force over all subsets, tie cases).   */
/* Per row: F = {kb : kb*bs < forced_tokens} is always kept; of the other    */
/* blocks the keep-|F| with the largest score are kept, equal scores going   */
/* to the lower block index.  The kept set is written sorted ascending.      */
/* row_ptr[r] = r*keep.  Scores must be finite.                              */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int64_t kb; } scored_block;

static int better(const scored_block *a, const scored_block *b) {
    if (a->s != b->s) return a->s > b->s;
    return a->kb < b->kb;
}

static int cmp_scored(const void *pa, const void *pb) {
    const scored_block *a = pa, *b = pb;
    if (better(a, b)) return -1;
    if (better(b, a)) return 1;
    return 0;
}

int orc_select_blocks(const double *s, int64_t rows, int64_t nkb, int64_t keep, int64_t bs,
                      int64_t forced_tokens, int32_t *row_ptr, int32_t *col_idx) {
    if (!s || !row_ptr || !col_idx || rows < 0 || nkb <= 0 || bs <= 0) return 1;
    int64_t forced = forced_tokens <= 0 ? 0 : (forced_tokens + bs - 1) / bs;
    if (forced > nkb) forced = nkb;
    if (keep < 1 || keep > nkb || forced > keep) return 2;
    scored_block *cand = malloc(sizeof(scored_block) * (size_t)nkb);
    unsigned char *kept = malloc((size_t)nkb);
    if (!cand || !kept) { free(cand); free(kept); return 3; }
    for (int64_t r = 0; r < rows; ++r) {
        const double *srow = s + r * nkb;
        memset(kept, 0, (size_t)nkb);
        for (int64_t kb = 0; kb < forced; ++kb) kept[kb] = 1;
        int64_t nc = 0;
        for (int64_t kb = forced; kb < nkb; ++kb) { cand[nc].s = srow[kb]; cand[nc].kb = kb; ++nc; }
        qsort(cand, (size_t)nc, sizeof(scored_block), cmp_scored);
        for (int64_t i = 0; i < keep - forced; ++i) kept[cand[i].kb] = 1;
        row_ptr[r] = (int32_t)(r * keep);
        int64_t pos = r * keep;
        for (int64_t kb = 0; kb < nkb; ++kb)
            if (kept[kb]) col_idx[pos++] = (int32_t)kb;
    }
    row_ptr[rows] = (int32_t)(rows * keep);
    free(cand);
    free(kept);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Shared problem description for the two attention steps.                  */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k, *v;   /* bf16 [bh][n][dpad] */
    int64_t bh_count, n, dpad, d, bs;
    double scale;
    const int32_t *row_ptr, *col_idx;  /* CSR over bh*nqb rows, head-local block ids */
    const int64_t *rows;         /* global row ids bh*n + i; NULL = all rows */
    int64_t nrows;
    /* capture outputs, per listed row */
    double *o, *m, *zf, *zk, *u;
    /* sparse inputs (may be NULL) and output */
    const double *cm, *czf, *czk, *cu;
    double *out;
    int mode;                    /* 0 = capture, 1 = sparse */
    int status;
} problem;

typedef struct { problem *p; int64_t begin, end; } work;

/* Mark, for query row i of head bh, which key blocks its query block keeps.
 * Returns 0 on success, nonzero if the CSR row is malformed. */
static int kept_blocks_of_row(const problem *p, int64_t bh, int64_t i, unsigned char *kept) {
    int64_t nkb = n_blocks_of(p->n, p->bs);
    int64_t r = bh * nkb + i / p->bs;
    memset(kept, 0, (size_t)nkb);
    for (int64_t e = p->row_ptr[r]; e < p->row_ptr[r + 1]; ++e) {
        int32_t kb = p->col_idx[e];
        if (kb < 0 || kb >= nkb) return 1;
        kept[kb] = 1;
    }
    return 0;
}

static double dot_qk(const problem *p, const uint16_t *qbase, int64_t bh, int64_t i,
                     const uint16_t *kbase, int64_t j) {
    const uint16_t *qr = qbase + (bh * p->n + i) * p->dpad;
    const uint16_t *kr = kbase + (bh * p->n + j) * p->dpad;
    double acc = 0.0;
    for (int64_t c = 0; c < p->d; ++c) acc += bf16_to_f64(qr[c]) * bf16_to_f64(kr[c]);
    return p->scale * acc;
}

/* Full-attention capture step for one row (pinned: torch SDPA in fp64,     */
/* rows sum to 1, Z_full = Z_kept + sum over masked, Z_full*O = Z_kept*O_kept */
/* + U, keep 100% gives U = 0 and Z_full = Z_kept).                          */
static void capture_row(problem *p, int64_t slot, int64_t g, double *s, unsigned char *kept) {
    int64_t bh = g / p->n, i = g % p->n, d = p->d;
    if (kept_blocks_of_row(p, bh, i, kept)) { p->status = 4; return; }
    double m = -INFINITY;
    for (int64_t j = 0; j < p->n; ++j) {
        s[j] = dot_qk(p, p->q, bh, i, p->k, j);
        if (s[j] > m) m = s[j];
    }
    double zf = 0.0, zk = 0.0;
    double *o = p->o + slot * d, *u = p->u + slot * d;
    for (int64_t c = 0; c < d; ++c) { o[c] = 0.0; u[c] = 0.0; }
    for (int64_t j = 0; j < p->n; ++j) {
        double e = exp(s[j] - m);
        int in_kept = kept[j / p->bs];
        const uint16_t *vr = p->v + (bh * p->n + j) * p->dpad;
        zf += e;
        if (in_kept) zk += e;
        for (int64_t c = 0; c < d; ++c) {
            double ev = e * bf16_to_f64(vr[c]);
            o[c] += ev;
            if (!in_kept) u[c] += ev;
        }
    }
    for (int64_t c = 0; c < d; ++c) o[c] /= zf;
    p->m[slot] = m;
    p->zf[slot] = zf;
    p->zk[slot] = zk;
}

/* Sparse step with statistical reshape for one row.  With cached stats:    */
/*   o = (N' + exp(m_c - m') * U) / (Z' * Z_full / Z_kept)                   */
/* where m', Z', N' run over the kept keys only; without stats o = N'/Z'.    */
/* A row whose query block keeps no key block gets o = 0.                    */
/* (pinned: keep 100% gives full attention of the current inputs; unchanged */
/* inputs give the capture step's full attention at any keep ratio; no      */
/* stats gives SDPA with a boolean block mask.)                              */
static void sparse_row(problem *p, int64_t slot, int64_t g, double *s, unsigned char *kept) {
    int64_t bh = g / p->n, i = g % p->n, d = p->d;
    double *out = p->out + slot * d;
    if (kept_blocks_of_row(p, bh, i, kept)) { p->status = 4; return; }
    double mp = -INFINITY;
    for (int64_t j = 0; j < p->n; ++j) {
        if (!kept[j / p->bs]) continue;
        s[j] = dot_qk(p, p->q, bh, i, p->k, j);
        if (s[j] > mp) mp = s[j];
    }
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    if (mp == -INFINITY) return;   /* empty kept set */
    double zp = 0.0;
    for (int64_t j = 0; j < p->n; ++j) {
        if (!kept[j / p->bs]) continue;
        double e = exp(s[j] - mp);
        const uint16_t *vr = p->v + (bh * p->n + j) * p->dpad;
        zp += e;
        for (int64_t c = 0; c < d; ++c) out[c] += e * bf16_to_f64(vr[c]);
    }
    if (p->cm) {
        double w = exp(p->cm[slot] - mp);
        double ratio = p->czf[slot] / p->czk[slot];
        const double *u = p->cu + slot * d;
        for (int64_t c = 0; c < d; ++c) out[c] = (out[c] + w * u[c]) / (zp * ratio);
    } else {
        for (int64_t c = 0; c < d; ++c) out[c] /= zp;
    }
}

static void *run_rows(void *arg) {
    work *w = arg;
    problem *p = w->p;
    double *s = malloc(sizeof(double) * (size_t)p->n);
    unsigned char *kept = malloc((size_t)n_blocks_of(p->n, p->bs));
    if (!s || !kept) { p->status = 3; free(s); free(kept); return NULL; }
    for (int64_t slot = w->begin; slot < w->end; ++slot) {
        int64_t g = p->rows ? p->rows[slot] : slot;
        if (g < 0 || g >= p->bh_count * p->n) { p->status = 5; continue; }
        if (p->mode == 0) capture_row(p, slot, g, s, kept);
        else sparse_row(p, slot, g, s, kept);
    }
    free(s);
    free(kept);
    return NULL;
}

static int run_parallel(problem *p, int threads) {
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if (threads > p->nrows) threads = p->nrows > 0 ? (int)p->nrows : 1;
    pthread_t tid[256];
    work w[256];
    int64_t per = (p->nrows + threads - 1) / threads;
    int started = 0;
    for (int t = 0; t < threads; ++t) {
        w[t].p = p;
        w[t].begin = t * per < p->nrows ? t * per : p->nrows;
        w[t].end = (t + 1) * per < p->nrows ? (t + 1) * per : p->nrows;
        if (threads == 1) { run_rows(&w[t]); continue; }
        if (pthread_create(&tid[t], NULL, run_rows, &w[t]) != 0) { run_rows(&w[t]); continue; }
        ++started;
        (void)started;
    }
    if (threads > 1)
        for (int t = 0; t < threads; ++t) pthread_join(tid[t], NULL);
    return p->status;
}

/* Full-attention capture step: per listed row, O_full[d], m, Z_full, Z_kept, U[d]. */
int orc_full_capture(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t bh_count,
                     int64_t n, int64_t dpad, int64_t d, int64_t bs, double scale,
                     const int32_t *row_ptr, const int32_t *col_idx, const int64_t *rows,
                     int64_t nrows, double *o, double *m, double *zf, double *zk, double *u,
                     int threads) {
    if (!q || !k || !v || !row_ptr || !col_idx || !o || !m || !zf || !zk || !u) return 1;
    if (n <= 0 || d <= 0 || dpad < d || bs <= 0 || bh_count < 0 || nrows < 0) return 1;
    problem p = {0};
    p.q = q; p.k = k; p.v = v; p.bh_count = bh_count; p.n = n; p.dpad = dpad; p.d = d;
    p.bs = bs; p.scale = scale; p.row_ptr = row_ptr; p.col_idx = col_idx;
    p.rows = rows; p.nrows = rows ? nrows : bh_count * n;
    p.o = o; p.m = m; p.zf = zf; p.zk = zk; p.u = u; p.mode = 0;
    return run_parallel(&p, threads);
}

/* Sparse step with reshape; cm/czf/czk/cu all NULL selects plain block-sparse attention. */
int orc_sparse_reshape(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t bh_count,
                       int64_t n, int64_t dpad, int64_t d, int64_t bs, double scale,
                       const int32_t *row_ptr, const int32_t *col_idx, const double *cm,
                       const double *czf, const double *czk, const double *cu,
                       const int64_t *rows, int64_t nrows, double *out, int threads) {
    if (!q || !k || !v || !row_ptr || !col_idx || !out) return 1;
    if (n <= 0 || d <= 0 || dpad < d || bs <= 0 || bh_count < 0 || nrows < 0) return 1;
    int nstats = (cm != NULL) + (czf != NULL) + (czk != NULL) + (cu != NULL);
    if (nstats != 0 && nstats != 4) return 1;
    problem p = {0};
    p.q = q; p.k = k; p.v = v; p.bh_count = bh_count; p.n = n; p.dpad = dpad; p.d = d;
    p.bs = bs; p.scale = scale; p.row_ptr = row_ptr; p.col_idx = col_idx;
    p.rows = rows; p.nrows = rows ? nrows : bh_count * n;
    p.cm = cm; p.czf = czf; p.czk = czk; p.cu = cu; p.out = out; p.mode = 1;
    return run_parallel(&p, threads);
}

/* ------------------------------------------------------------------------ */
/* Exact block attention mass (pinned: rows of a query block sum to its     */
/* token count; uniform scores give rows*cols/n; brute force against torch  */
/* softmax in fp64 summed over the blocks).                                  */
/* mass[bh][qb][kb] = sum over query tokens i of block qb (i < n) and key   */
/* tokens j of block kb (j < n) of softmax_j(scale * q_i . k_j), the        */
/* softmax taken over all n keys of row i.  Selecting the top-k of these    */
/* per query block (orc_select_blocks) keeps the key blocks that carry the  */
/* most attention probability in the step they are computed from.          */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k;
    int64_t bh_count, n, dpad, d, bs;
    double scale;
    double *mass;
    const int64_t *qblocks;      /* listed query-block ids bh*nb + qb; NULL = all */
    int64_t begin, end;          /* slots handled by this worker */
    int status;
} mass_work;

static void *mass_rows(void *arg) {
    mass_work *w = arg;
    int64_t nb = n_blocks_of(w->n, w->bs);
    problem p = {0};             /* for dot_qk only */
    p.n = w->n; p.dpad = w->dpad; p.d = w->d; p.scale = w->scale;
    double *s = malloc(sizeof(double) * (size_t)w->n);
    if (!s) { w->status = 3; return NULL; }
    for (int64_t slot = w->begin; slot < w->end; ++slot) {
        int64_t r = w->qblocks ? w->qblocks[slot] : slot;
        if (r < 0 || r >= w->bh_count * nb) { w->status = 5; continue; }
        int64_t bh = r / nb, qb = r % nb;
        double *out = w->mass + slot * nb;
        for (int64_t kb = 0; kb < nb; ++kb) out[kb] = 0.0;
        int64_t i1 = (qb + 1) * w->bs < w->n ? (qb + 1) * w->bs : w->n;
        for (int64_t i = qb * w->bs; i < i1; ++i) {
            double m = -INFINITY, z = 0.0;
            for (int64_t j = 0; j < w->n; ++j) {
                s[j] = dot_qk(&p, w->q, bh, i, w->k, j);
                if (s[j] > m) m = s[j];
            }
            for (int64_t j = 0; j < w->n; ++j) z += exp(s[j] - m);
            for (int64_t j = 0; j < w->n; ++j) out[j / w->bs] += exp(s[j] - m) / z;
        }
    }
    free(s);
    return NULL;
}

/* mass is [nq][nb] for the listed query blocks (qblocks), [bh*nb][nb] when qblocks is NULL. */
int orc_block_mass(const uint16_t *q, const uint16_t *k, int64_t bh_count, int64_t n, int64_t dpad,
                   int64_t d, int64_t bs, double scale, const int64_t *qblocks, int64_t nq, double *mass,
                   int threads) {
    if (!q || !k || !mass || n <= 0 || d <= 0 || dpad < d || bs <= 0 || bh_count < 0 || nq < 0) return 1;
    int64_t rows = qblocks ? nq : bh_count * n_blocks_of(n, bs);
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if (threads > rows) threads = rows > 0 ? (int)rows : 1;
    pthread_t tid[256];
    mass_work w[256];
    int64_t per = (rows + threads - 1) / threads;
    int status = 0;
    for (int t = 0; t < threads; ++t) {
        w[t] = (mass_work){q, k, bh_count, n, dpad, d, bs, scale, mass, qblocks, 0, 0, 0};
        w[t].begin = t * per < rows ? t * per : rows;
        w[t].end = (t + 1) * per < rows ? (t + 1) * per : rows;
        if (threads == 1 || pthread_create(&tid[t], NULL, mass_rows, &w[t]) != 0) {
            mass_rows(&w[t]);
            tid[t] = 0;
        }
    }
    for (int t = 0; t < threads; ++t)
        if (threads > 1 && tid[t]) pthread_join(tid[t], NULL);
    for (int t = 0; t < threads; ++t)
        if (w[t].status) status = w[t].status;
    return status;
}
