/*
 * art_oracle.h -- CPU oracle for ART run-time-terminated decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this code.  It shares no source,
 * header, table or helper with the CUDA library and includes nothing from it.
 *
 * What it computes (ART: Attention Run-time Termination, "2. Methodology"):
 * single-token decode attention over a paged K/V cache, walked block by block
 * in a caller-given order (section 2.4, "reordering the traversal sequence of
 * KV blocks"), with an online-softmax state updated after each block
 * (section 2.1, streaming tile-wise accumulation).  After every block after
 * the first, two statistics of the partial output o_j against o_{j-1} are
 * compared with thresholds (section 2.2): the relative magnitude change
 * |‖o_j‖-‖o_{j-1}‖|/‖o_{j-1}‖ < eps_m and the direction change
 * 1-cos(o_j, o_{j-1}) < eps_d.  A patience counter counts consecutive blocks
 * on which both hold and resets otherwise (section 2.3).  The walk stops
 * after the block that brings the counter to P, provided at least min_blocks
 * blocks were consumed; block 0 of the walk is always consumed (section 2.4,
 * attention sinks).  Everything is computed in IEEE double precision.
 *
 * Because the stop index is a discrete decision taken on floating-point
 * statistics, the oracle also reports the set of stop indices that are
 * admissible when every comparison whose statistic lies within `band`
 * (relative) of its threshold is allowed to go either way.
 */
#ifndef ART_ORACLE_H
#define ART_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type codes of the cache and query arrays. */
#define ART_ORACLE_F32  0   /* IEEE binary32                              */
#define ART_ORACLE_BF16 1   /* bfloat16 stored as raw 16-bit patterns     */

typedef struct {
    int32_t dtype;                  /* ART_ORACLE_F32 or ART_ORACLE_BF16            */
    int32_t B, Hq, Hkv, d, page;    /* batch, query heads, kv heads, head dim, block */
    int32_t max_blocks;             /* columns of page_table / block_order          */
    int32_t num_pages;              /* first dimension of the caches                */
    const void *q;                  /* [B][Hq][d]                                   */
    int64_t q_stride[3];            /* element strides of q                         */
    const void *k;                  /* [num_pages][Hkv][page][d]                    */
    int64_t k_stride[4];
    const void *v;                  /* same shape as k                              */
    int64_t v_stride[4];
    const int32_t *page_table;      /* [B][max_blocks] physical page of logical blk */
    const int32_t *block_order;     /* [B][max_blocks] logical block at walk step j */
    const int32_t *seq_lens;        /* [B]                                          */
    double scale;                   /* softmax scale, normally 1/sqrt(d)            */
    const double *eps_m;            /* [B] magnitude threshold                      */
    const double *eps_d;            /* [B] direction threshold                      */
    const int32_t *P;               /* [B] patience                                 */
    const int32_t *min_blocks;      /* [B]                                          */
    double band;                    /* relative half-width of the ambiguity band    */
} art_oracle_problem;

typedef struct {
    int32_t *stop;        /* [B*Hkv] canonical stop (blocks consumed)                */
    int32_t *adm_count;   /* [B*Hkv] number of admissible stops                      */
    int32_t *adm;         /* [B*Hkv][adm_cap] admissible stops, ascending            */
    int32_t adm_cap;      /* capacity per unit of adm (entries beyond are dropped)   */
    int32_t *amb_count;   /* [B*Hkv] blocks whose stable flag was undetermined       */
    double *out;          /* [B][Hq][d] output at the canonical stop, or NULL        */
    double *ds;           /* [B*Hkv][max_blocks] magnitude statistic or NULL         */
    double *dd;           /* [B*Hkv][max_blocks] direction statistic or NULL         */
    int8_t *flag;         /* [B*Hkv][max_blocks] 'T','F','?' (0 at j=0/unused) or NULL */
} art_oracle_result;

/* Status codes. */
#define ART_ORACLE_OK        0
#define ART_ORACLE_EINVAL   -1   /* inconsistent sizes or NULL required pointer */
#define ART_ORACLE_EINDEX   -2   /* an order/page entry out of range             */
#define ART_ORACLE_ENOMEM   -3

/* Run the walk for every (b, kv-head) unit.  nthreads <= 0 uses all cores. */
int art_oracle_run(const art_oracle_problem *prob, art_oracle_result *res, int nthreads);

/* Output after the first s[i] blocks of the walk of unit units[i] (unit =
 * b*Hkv + h): out[i][g][k] for the G = Hq/Hkv query heads of the unit.
 * s[i] = 0 gives zeros. */
int art_oracle_prefix_out(const art_oracle_problem *prob, int32_t nsel, const int32_t *units,
                          const int32_t *s, double *out, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
