/*
 * art_oracle.c -- plain, slow CPU oracle for ART run-time-terminated decode
 * attention.  TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and
 * the benchmark's CPU-baseline leg are its only users; the product library
 * never links or calls it, and it shares no code with the CUDA path.
 *
 * Source of the method: "ART: Attention Run-time Termination for Efficient
 * Large Language Model Decoding" (gist.science explainer), Technical Summary
 * section 2 -- 2.1 streaming tile-wise accumulation of the attention output,
 * 2.2 the two stability statistics and their thresholds, 2.3 the patience
 * counter, 2.4 traversal reordering and the mandatory sink block.  The
 * statistics used here are the full-vector relative magnitude change and one
 * minus the cosine, both compared with a strict "<"; the explainer words
 * them as "L2-norm difference" and "cosine similarity deviation" of a probe
 * vector.
 *
 * Arithmetic: every input value is upcast exactly to double; all sums,
 * exponentials and statistics are double precision; no blocking, fusion or
 * reordering beyond the per-block online-softmax update the method itself
 * prescribes.  Statistics use their plain definitions.
 */
#include "art_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ---- input access ------------------------------------------------------ */

static double load_elem(int32_t dtype, const void *base, int64_t idx)
{
    if (dtype == ART_ORACLE_F32)
        return (double)((const float *)base)[idx];
    /* bfloat16: the 16 stored bits are the top half of an IEEE binary32 */
    uint32_t w = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static int64_t n_blocks_of(const art_oracle_problem *p, int b)
{
    int64_t L = p->seq_lens[b];
    if (L <= 0)
        return 0;
    return (L + p->page - 1) / p->page;
}

/* ---- one unit's walk ---------------------------------------------------- */

typedef struct {
    int G, d, page;
    double *q;      /* [G][d]    query heads of the unit                    */
    double *acc;    /* [G][d]    unnormalised running numerator             */
    double *m;      /* [G]       running maximum score                      */
    double *l;      /* [G]       running denominator                        */
    double *s;      /* [G][page] scores of the current block                */
    double *o;      /* [G*d]     normalised output after the current block  */
    double *o_prev; /* [G*d]     normalised output after the previous block */
    uint8_t *seen;  /* [max_blocks] permutation check                        */
    uint8_t *states;/* [P+1] set-valued counter for the admissible stops     */
    uint8_t *states_next;
} walk_ws;

static void ws_free(walk_ws *w)
{
    free(w->q); free(w->acc); free(w->m); free(w->l); free(w->s);
    free(w->o); free(w->o_prev); free(w->seen); free(w->states); free(w->states_next);
    memset(w, 0, sizeof *w);
}

static int ws_alloc(walk_ws *w, const art_oracle_problem *p, int32_t maxP)
{
    memset(w, 0, sizeof *w);
    w->G = p->Hq / p->Hkv;
    w->d = p->d;
    w->page = p->page;
    size_t gd = (size_t)w->G * w->d;
    w->q = malloc(gd * sizeof(double));
    w->acc = malloc(gd * sizeof(double));
    w->m = malloc(w->G * sizeof(double));
    w->l = malloc(w->G * sizeof(double));
    w->s = malloc((size_t)w->G * w->page * sizeof(double));
    w->o = malloc(gd * sizeof(double));
    w->o_prev = malloc(gd * sizeof(double));
    w->seen = malloc((size_t)p->max_blocks + 1);
    w->states = malloc((size_t)maxP + 2);
    w->states_next = malloc((size_t)maxP + 2);
    if (!w->q || !w->acc || !w->m || !w->l || !w->s || !w->o || !w->o_prev || !w->seen || !w->states || !w->states_next) {
        ws_free(w);
        return ART_ORACLE_ENOMEM;
    }
    return ART_ORACLE_OK;
}

/* Reset the online-softmax state: m = -inf, l = 0, acc = 0 (section 2.1). */
static void state_reset(walk_ws *w, const art_oracle_problem *p, int b, int h)
{
    for (int g = 0; g < w->G; ++g) {
        int hq = h * w->G + g;  /* query head hq reads kv head hq / G */
        for (int k = 0; k < w->d; ++k)
            w->q[g * w->d + k] = load_elem(p->dtype, p->q,
                (int64_t)b * p->q_stride[0] + (int64_t)hq * p->q_stride[1] + (int64_t)k * p->q_stride[2]);
        w->m[g] = -INFINITY;
        w->l[g] = 0.0;
        for (int k = 0; k < w->d; ++k)
            w->acc[g * w->d + k] = 0.0;
    }
}

/* Fold walk step j into the online-softmax state.  Returns 0 or EINDEX. */
static int state_add_block(walk_ws *w, const art_oracle_problem *p, int b, int h, int64_t j, int64_t N)
{
    int32_t lb = p->block_order[(int64_t)b * p->max_blocks + j];
    if (lb < 0 || lb >= N)
        return ART_ORACLE_EINDEX;
    int32_t pp = p->page_table[(int64_t)b * p->max_blocks + lb];
    if (pp < 0 || pp >= p->num_pages)
        return ART_ORACLE_EINDEX;
    int64_t L = p->seq_lens[b];
    int64_t kbase = (int64_t)pp * p->k_stride[0] + (int64_t)h * p->k_stride[1];
    int64_t vbase = (int64_t)pp * p->v_stride[0] + (int64_t)h * p->v_stride[1];

    for (int g = 0; g < w->G; ++g) {
        /* scores s_t = scale * q . k_t for the block's tokens inside the sequence */
        double smax = -INFINITY;
        for (int t = 0; t < w->page; ++t) {
            int64_t pos = (int64_t)lb * w->page + t;
            if (pos >= L) {
                w->s[g * w->page + t] = -INFINITY;   /* past the end: masked */
                continue;
            }
            double dot = 0.0;
            for (int k = 0; k < w->d; ++k)
                dot += w->q[g * w->d + k] *
                       load_elem(p->dtype, p->k, kbase + (int64_t)t * p->k_stride[2] + (int64_t)k * p->k_stride[3]);
            double s = p->scale * dot;
            w->s[g * w->page + t] = s;
            if (s > smax)
                smax = s;
        }
        if (smax == -INFINITY)
            continue;   /* no token of this block is inside the sequence */
        /* m' = max(m, max_t s_t); l = l e^{m-m'} + sum e^{s-m'}; acc likewise */
        double mnew = w->m[g] > smax ? w->m[g] : smax;
        double alpha = (w->m[g] == -INFINITY) ? 0.0 : exp(w->m[g] - mnew);
        w->l[g] *= alpha;
        for (int k = 0; k < w->d; ++k)
            w->acc[g * w->d + k] *= alpha;
        for (int t = 0; t < w->page; ++t) {
            double s = w->s[g * w->page + t];
            if (s == -INFINITY)
                continue;
            double e = exp(s - mnew);
            w->l[g] += e;
            for (int k = 0; k < w->d; ++k)
                w->acc[g * w->d + k] += e *
                    load_elem(p->dtype, p->v, vbase + (int64_t)t * p->v_stride[2] + (int64_t)k * p->v_stride[3]);
        }
        w->m[g] = mnew;
    }
    return ART_ORACLE_OK;
}

/* o = concat_g(acc_g / l_g): the partial attention output, length G*d. */
static void state_output(walk_ws *w, double *o)
{
    for (int g = 0; g < w->G; ++g)
        for (int k = 0; k < w->d; ++k)
            o[g * w->d + k] = (w->l[g] > 0.0) ? w->acc[g * w->d + k] / w->l[g] : 0.0;
}

/* Three-valued "x < eps": 'T', 'F', or '?' when x lies within band*eps of a
 * positive finite threshold.  eps = 0 never passes (the statistics are >= 0);
 * eps = +inf always passes for a finite statistic. */
static char cmp3(double x, double eps, double band)
{
    if (!(eps > 0.0))
        return 'F';
    if (isinf(eps))
        return isfinite(x) ? 'T' : 'F';
    if (fabs(x - eps) <= band * eps)
        return '?';
    return x < eps ? 'T' : 'F';
}

static char and3(char a, char b)
{
    if (a == 'F' || b == 'F')
        return 'F';
    if (a == '?' || b == '?')
        return '?';
    return 'T';
}

static int check_order_is_permutation(walk_ws *w, const art_oracle_problem *p, int b, int64_t N)
{
    memset(w->seen, 0, (size_t)p->max_blocks + 1);
    for (int64_t j = 0; j < N; ++j) {
        int32_t lb = p->block_order[(int64_t)b * p->max_blocks + j];
        if (lb < 0 || lb >= N || w->seen[lb])
            return ART_ORACLE_EINDEX;
        w->seen[lb] = 1;
    }
    return ART_ORACLE_OK;
}

static void adm_add(const art_oracle_result *r, int64_t unit, int32_t stop)
{
    int32_t n = r->adm_count[unit];
    if (n > 0 && r->adm[unit * r->adm_cap + n - 1] == stop)
        return;  /* stops are produced in ascending order */
    if (n < r->adm_cap)
        r->adm[unit * r->adm_cap + n] = stop;
    r->adm_count[unit] = n + 1;
}

/* The ART walk of unit (b, h) with the stop rule. */
static int run_unit(walk_ws *w, const art_oracle_problem *p, const art_oracle_result *r, int b, int h)
{
    int64_t unit = (int64_t)b * p->Hkv + h;
    int64_t N = n_blocks_of(p, b);
    int G = w->G, d = w->d;
    int32_t P = p->P[b], minb = p->min_blocks[b];
    double eps_m = p->eps_m[b], eps_d = p->eps_d[b];

    r->adm_count[unit] = 0;
    r->amb_count[unit] = 0;
    if (r->ds)
        for (int64_t j = 0; j < p->max_blocks; ++j) {
            r->ds[unit * p->max_blocks + j] = NAN;
            r->dd[unit * p->max_blocks + j] = NAN;
        }
    if (r->flag)
        memset(r->flag + unit * p->max_blocks, 0, (size_t)p->max_blocks);

    if (N == 0) {  /* empty sequence: nothing to read, output zero */
        r->stop[unit] = 0;
        adm_add(r, unit, 0);
        if (r->out)
            for (int g = 0; g < G; ++g)
                for (int k = 0; k < d; ++k)
                    r->out[((int64_t)b * p->Hq + h * G + g) * d + k] = 0.0;
        return ART_ORACLE_OK;
    }
    int rc = check_order_is_permutation(w, p, b, N);
    if (rc)
        return rc;

    state_reset(w, p, b, h);
    int32_t c = 0;             /* canonical patience counter */
    int32_t stop = -1;         /* canonical stop once found  */
    memset(w->states, 0, (size_t)P + 2);
    w->states[0] = 1;          /* set of live counter values for the admissible stops */
    int live = 1;

    for (int64_t j = 0; j < N && (stop < 0 || live); ++j) {
        rc = state_add_block(w, p, b, h, j, N);
        if (rc)
            return rc;
        state_output(w, w->o);

        if (j >= 1) {
            /* statistics of o_j against o_{j-1}: plain definitions */
            double n1 = 0.0, n0 = 0.0, dot = 0.0;
            for (int i = 0; i < G * d; ++i) {
                n1 += w->o[i] * w->o[i];
                n0 += w->o_prev[i] * w->o_prev[i];
                dot += w->o[i] * w->o_prev[i];
            }
            n1 = sqrt(n1);
            n0 = sqrt(n0);
            char flag;
            int canon_stable;
            if (n0 == 0.0 || n1 == 0.0) {
                flag = 'F';        /* no direction to compare: never stable */
                canon_stable = 0;
            } else {
                double dscale = fabs(n1 - n0) / n0;
                double ddir = 1.0 - dot / (n1 * n0);
                if (ddir < 0.0)
                    ddir = 0.0;
                if (r->ds) {
                    r->ds[unit * p->max_blocks + j] = dscale;
                    r->dd[unit * p->max_blocks + j] = ddir;
                }
                flag = and3(cmp3(dscale, eps_m, p->band), cmp3(ddir, eps_d, p->band));
                canon_stable = (dscale < eps_m) && (ddir < eps_d);
            }
            if (r->flag)
                r->flag[unit * p->max_blocks + j] = (int8_t)flag;
            if (flag == '?')
                r->amb_count[unit] += 1;

            /* patience (section 2.3): consecutive stable blocks */
            c = canon_stable ? c + 1 : 0;

            /* the same counter over the set of outcomes the band allows:
             * 'T' maps c -> min(c+1, P), 'F' maps c -> 0, '?' maps c to both */
            if (live) {
                uint8_t *S = w->states, *T = w->states_next;
                memset(T, 0, (size_t)P + 1);
                for (int32_t v = 0; v <= P; ++v) {
                    if (!S[v])
                        continue;
                    if (flag == 'T' || flag == '?')
                        T[v + 1 > P ? P : v + 1] = 1;
                    if (flag == 'F' || flag == '?')
                        T[0] = 1;
                }
                memcpy(S, T, (size_t)P + 1);
            }
        }

        /* stop test after consuming j+1 blocks */
        if (stop < 0 && c >= P && j + 1 >= minb) {
            stop = (int32_t)(j + 1);
            if (r->out)
                for (int g = 0; g < G; ++g)
                    for (int k = 0; k < d; ++k)
                        r->out[((int64_t)b * p->Hq + h * G + g) * d + k] = w->o[g * d + k];
        }
        if (live) {
            live = 0;
            for (int32_t v = 0; v <= P; ++v) {
                if (!w->states[v])
                    continue;
                if (v >= P && j + 1 >= minb) {
                    adm_add(r, unit, (int32_t)(j + 1));
                    w->states[v] = 0;
                } else {
                    live = 1;
                }
            }
        }
        memcpy(w->o_prev, w->o, (size_t)G * d * sizeof(double));
    }
    if (stop < 0) {  /* walked every block */
        stop = (int32_t)N;
        if (r->out)
            for (int g = 0; g < G; ++g)
                for (int k = 0; k < d; ++k)
                    r->out[((int64_t)b * p->Hq + h * G + g) * d + k] = w->o[g * d + k];
    }
    if (live)
        adm_add(r, unit, (int32_t)N);
    r->stop[unit] = stop;
    return ART_ORACLE_OK;
}

/* ---- validation ------------------------------------------------------------ */

static int validate(const art_oracle_problem *p)
{
    if (!p || !p->q || !p->k || !p->v || !p->page_table || !p->block_order || !p->seq_lens)
        return ART_ORACLE_EINVAL;
    if (p->dtype != ART_ORACLE_F32 && p->dtype != ART_ORACLE_BF16)
        return ART_ORACLE_EINVAL;
    if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv || p->d <= 0 || p->page <= 0 ||
        p->max_blocks <= 0 || p->num_pages <= 0)
        return ART_ORACLE_EINVAL;
    for (int b = 0; b < p->B; ++b)
        if ((int64_t)p->seq_lens[b] > (int64_t)p->max_blocks * p->page)
            return ART_ORACLE_EINVAL;
    return ART_ORACLE_OK;
}

static int validate_rule(const art_oracle_problem *p, int32_t *maxP)
{
    if (!p->eps_m || !p->eps_d || !p->P || !p->min_blocks)
        return ART_ORACLE_EINVAL;
    *maxP = 0;
    for (int b = 0; b < p->B; ++b) {
        if (p->P[b] < 0 || p->min_blocks[b] < 0 || isnan(p->eps_m[b]) || isnan(p->eps_d[b]) ||
            p->eps_m[b] < 0 || p->eps_d[b] < 0)
            return ART_ORACLE_EINVAL;
        if (p->P[b] > *maxP)
            *maxP = p->P[b];
    }
    return ART_ORACLE_OK;
}

/* ---- thread pool over units ------------------------------------------------ */

typedef struct {
    const art_oracle_problem *p;
    const art_oracle_result *r;
    int32_t nsel;
    const int32_t *units, *s;
    double *out;
    int32_t maxP;
    int mode;                 /* 0: stop rule, 1: prefix outputs */
    atomic_long next;
    atomic_int status;
} pool_job;

static int prefix_one(walk_ws *w, const art_oracle_problem *p, int32_t unit, int32_t s, double *out)
{
    int b = unit / p->Hkv, h = unit % p->Hkv;
    int64_t N = n_blocks_of(p, b);
    if (s < 0 || s > N)
        return ART_ORACLE_EINVAL;
    if (N > 0) {
        int rc = check_order_is_permutation(w, p, b, N);
        if (rc)
            return rc;
    }
    state_reset(w, p, b, h);
    for (int64_t j = 0; j < s; ++j) {
        int rc = state_add_block(w, p, b, h, j, N);
        if (rc)
            return rc;
    }
    state_output(w, out);
    return ART_ORACLE_OK;
}

static void *pool_worker(void *arg)
{
    pool_job *job = arg;
    walk_ws w;
    if (ws_alloc(&w, job->p, job->maxP)) {
        atomic_store(&job->status, ART_ORACLE_ENOMEM);
        return NULL;
    }
    const art_oracle_problem *p = job->p;
    long total = job->mode == 0 ? (long)p->B * p->Hkv : job->nsel;
    for (;;) {
        long i = atomic_fetch_add(&job->next, 1);
        if (i >= total || atomic_load(&job->status) != ART_ORACLE_OK)
            break;
        int rc;
        if (job->mode == 0)
            rc = run_unit(&w, p, job->r, (int)(i / p->Hkv), (int)(i % p->Hkv));
        else
            rc = prefix_one(&w, p, job->units[i], job->s[i], job->out + i * (int64_t)w.G * w.d);
        if (rc) {
            int expect = ART_ORACLE_OK;
            atomic_compare_exchange_strong(&job->status, &expect, rc);
        }
    }
    ws_free(&w);
    return NULL;
}

static int run_pool(pool_job *job, int nthreads, long total)
{
    if (nthreads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = n > 0 ? (int)n : 1;
    }
    if (nthreads > total)
        nthreads = total > 0 ? (int)total : 1;
    atomic_store(&job->next, 0);
    atomic_store(&job->status, ART_ORACLE_OK);
    if (nthreads == 1) {
        pool_worker(job);
        return atomic_load(&job->status);
    }
    pthread_t *tid = malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!tid)
        return ART_ORACLE_ENOMEM;
    int started = 0;
    for (; started < nthreads; ++started)
        if (pthread_create(&tid[started], NULL, pool_worker, job))
            break;
    if (started == 0) {
        free(tid);
        pool_worker(job);
        return atomic_load(&job->status);
    }
    for (int i = 0; i < started; ++i)
        pthread_join(tid[i], NULL);
    free(tid);
    return atomic_load(&job->status);
}

int art_oracle_run(const art_oracle_problem *p, art_oracle_result *r, int nthreads)
{
    int rc = validate(p);
    if (rc)
        return rc;
    int32_t maxP;
    rc = validate_rule(p, &maxP);
    if (rc)
        return rc;
    if (!r || !r->stop || !r->adm_count || !r->adm || r->adm_cap <= 0 || !r->amb_count ||
        (!r->ds) != (!r->dd))
        return ART_ORACLE_EINVAL;
    pool_job job;
    memset(&job, 0, sizeof job);
    job.p = p;
    job.r = r;
    job.maxP = maxP;
    job.mode = 0;
    return run_pool(&job, nthreads, (long)p->B * p->Hkv);
}

int art_oracle_prefix_out(const art_oracle_problem *p, int32_t nsel, const int32_t *units,
                          const int32_t *s, double *out, int nthreads)
{
    int rc = validate(p);
    if (rc)
        return rc;
    if (nsel < 0 || (nsel > 0 && (!units || !s || !out)))
        return ART_ORACLE_EINVAL;
    for (int32_t i = 0; i < nsel; ++i)
        if (units[i] < 0 || units[i] >= p->B * p->Hkv)
            return ART_ORACLE_EINVAL;
    pool_job job;
    memset(&job, 0, sizeof job);
    job.p = p;
    job.nsel = nsel;
    job.units = units;
    job.s = s;
    job.out = out;
    job.mode = 1;
    return run_pool(&job, nthreads, nsel);
}
