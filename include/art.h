/*
 * art.h -- C ABI of libart, B200 (sm_100a) ART run-time-terminated decode
 * attention.
 *
 * Method: "ART: Attention Run-time Termination for Efficient Large Language
 * Model Decoding" (gist.science explainer), Technical Summary, section 2.
 * One decode step of one attention layer: each sequence's single query token
 * attends over its paged K/V cache.  The cache of each (sequence, kv-head)
 * unit is walked one block (= one page) at a time in a caller-given order
 * (section 2.4, traversal reordering), keeping an online-softmax state
 * (section 2.1).  After every block j >= 1 the partial output o_j (the G
 * query heads of the unit, concatenated) is compared with o_{j-1}:
 *
 *     d_scale = | ||o_j|| - ||o_{j-1}|| | / ||o_{j-1}||      stable if < eps_m
 *     d_dir   = 1 - cos(o_j, o_{j-1})                      stable if < eps_d
 *
 * (section 2.2: both must hold).  A patience counter counts consecutive
 * stable blocks and resets on an unstable one (section 2.3).  The walk stops
 * after the block that brings the counter to P, once at least min_blocks
 * blocks were consumed; the first block of the order is always consumed
 * (section 2.4, attention sinks).  The blocks after the stop are never
 * fetched from HBM.  eps = 0 disables termination (full attention).
 *
 * Conventions for every entry point:
 *  - Tensors are described by art_tensor_t: a DEVICE pointer owned by the
 *    caller, an element type, and shape/stride in ELEMENTS.  The library
 *    never allocates, frees or retains them.
 *  - Calls are asynchronous on the given stream (NULL = legacy default
 *    stream): the results are valid once the stream has reached the call.
 *  - All argument checks happen on the host, before any CUDA call; a failed
 *    check returns its status and launches nothing.
 *  - Errors found on the device (an order or page-table entry out of range,
 *    a sequence longer than max_blocks pages, an expired wait) never trap:
 *    the affected unit gets stop_block = -1 and, when the caller passes
 *    device_status, the first such error code is stored there.
 */
#ifndef ART_H
#define ART_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *art_stream_t;   /* a cudaStream_t */

typedef enum {
    ART_F32 = 0,    /* IEEE binary32                */
    ART_BF16 = 1,   /* bfloat16                     */
    ART_I32 = 2     /* int32                        */
} art_dtype_t;

typedef struct {
    void *data;          /* device pointer (caller-owned)                    */
    int32_t dtype;       /* art_dtype_t                                      */
    int32_t ndim;        /* number of valid entries in shape/stride          */
    int64_t shape[4];
    int64_t stride[4];   /* in elements                                      */
} art_tensor_t;

typedef enum {
    ART_OK = 0,
    ART_ERR_NULL = -1,           /* a required pointer is NULL                           */
    ART_ERR_SHAPE = -2,          /* inconsistent shapes, strides or alignment            */
    ART_ERR_DTYPE = -3,          /* wrong or mismatched element type                     */
    ART_ERR_UNSUPPORTED = -4,    /* head dim, page size or group size not compiled       */
    ART_ERR_PARAM = -5,          /* eps < 0 or NaN, P < 0, min_blocks < 0, bad option    */
    ART_ERR_LAUNCH = -6,         /* the CUDA runtime refused the launch                  */
    ART_ERR_DEVICE_TIMEOUT = -7, /* (device_status) a bounded wait expired               */
    ART_ERR_BAD_INDEX = -8,      /* (device_status) order/page entry or length invalid   */
    ART_ERR_SCRATCH_SIZE = -9    /* art_decode_attention_no_alloc: the problem needs     */
                                 /* more than ART_NO_ALLOC_SCRATCH_BYTES of scratch      */
} art_status_t;

/*
 * art_decode_attention -- one ART decode-attention step.
 *
 *  q           [B, Hq, d]                     F32 or BF16; d contiguous.
 *  k_cache     [num_pages, Hkv, page, d]      same type as q; d contiguous; the other
 *                                             strides multiples of 16 bytes, base 16-byte
 *                                             aligned (the cache is read with TMA).
 *  v_cache     same shape and type as k_cache (strides may differ).
 *  page_table  [B, max_blocks] I32: physical page of logical block lb of sequence b.
 *  block_order [B, max_blocks] I32: logical block visited at walk step j; entries
 *                                   0..N_b-1 must be a permutation of 0..N_b-1 where
 *                                   N_b = ceil(seq_lens[b] / page).  An entry out
 *                                   of [0, N_b) is reported (ART_ERR_BAD_INDEX); a
 *                                   repeated or missing block is not detected (the
 *                                   walk would fold one block twice and skip
 *                                   another: the result is undefined).  Entries past
 *                                   N_b are never read.  May be NULL (or have NULL
 *                                   data): the walk then takes the default order
 *                                   [0, N_b-1, ..., 1] (sink block, then newest to
 *                                   oldest), computed on the fly.
 *  seq_lens    [B] I32 (contiguous): tokens in the cache of sequence b.  Token
 *                                   lb*page + t of the sequence is row t of page
 *                                   page_table[b, lb]; rows past seq_lens[b] are masked.
 *  eps_m, eps_d  thresholds (>= 0, not NaN; 0 disables, +inf always passes).
 *  P           patience (>= 0).  min_blocks: lower bound on blocks consumed (>= 0).
 *  out         [B, Hq, d] F32: attention output at the stop (0 for empty sequences).
 *  stop_block  [B, Hkv] I32: blocks consumed by the walk (0 for empty sequences,
 *                            -1 for a unit that hit a device-side error).
 * Query head i uses kv head i / (Hq / Hkv).  The softmax scale is 1/sqrt(d).
 * Supported: d in {64, 128}; page in {16, 64}; Hq/Hkv in 1..8.
 */
art_status_t art_decode_attention(const art_tensor_t *q, const art_tensor_t *k_cache,
                                  const art_tensor_t *v_cache, const art_tensor_t *page_table,
                                  const art_tensor_t *block_order, const art_tensor_t *seq_lens,
                                  float eps_m, float eps_d, int32_t P, int32_t min_blocks,
                                  art_tensor_t *out, art_tensor_t *stop_block, art_stream_t stream);

/* What art_decode_attention_ex chose; filled when art_params_t.info != NULL. */
typedef struct {
    int32_t engine;        /* 1 = CUDA-core block engine, 2 = tensor-core (mma) engine   */
    int32_t cluster_size;  /* CTAs cooperating on one (sequence, kv-head) unit           */
    int32_t grid;          /* CTAs launched                                               */
    int32_t threads;       /* threads per CTA                                             */
    int32_t stages;        /* K/V pages buffered per CTA                                  */
    int32_t compute_warps; /* warps turning pages into block states, per CTA              */
    int32_t window;        /* blocks fetched ahead of the merged prefix (the bound on      */
                           /* pages read past the stop)                                    */
    int32_t smem_bytes;    /* dynamic shared memory per CTA                               */
    int32_t prefetch;      /* further blocks pulled into L2 ahead of the staged ones      */
    int32_t merge_cta;     /* 1: the cluster's first CTA only merges; 2: one merge CTA    */
                           /* per unit reached through the workspace                      */
    int32_t ring_slots;    /* block states the merging CTA holds (= window, or fewer with */
                           /* merge_cta: then a finished state waits for a free slot)     */
} art_launch_info_t;

typedef struct {
    art_tensor_t q, k_cache, v_cache, page_table, block_order, seq_lens, out, stop_block;
    float eps_m, eps_d;            /* used where the per-sequence arrays are NULL           */
    int32_t P, min_blocks;
    float sm_scale;                /* softmax scale; <= 0 selects 1/sqrt(d)                 */
    const float *eps_m_per_seq;    /* device [B] or NULL                                    */
    const float *eps_d_per_seq;    /* device [B] or NULL                                    */
    const int32_t *P_per_seq;      /* device [B] or NULL                                    */
    const int32_t *min_blocks_per_seq; /* device [B] or NULL                                */
    int32_t *blocks_fetched;       /* device [B*Hkv] or NULL: pages whose fetch was issued  */
    int32_t *device_status;        /* device [1] or NULL: first device-side error (0 = ok); */
                                   /* the caller zeroes it; the library only writes errors  */
    int32_t engine;                /* 0 auto, 1 CUDA cores (any dtype), 2 tensor cores (BF16)*/
    int32_t cluster_size;          /* 0 auto, else 1..16 CTAs per unit                      */
    int32_t stages;                /* 0 auto, else 2..8 (a multiple of compute_warps)       */
    int32_t compute_warps;         /* 0 auto, else 1..6                                     */
    int32_t window;                /* 0 auto, else 8..128 blocks fetched ahead of the       */
                                   /* merged prefix (speculation; pages read past the stop  */
                                   /* stay below it).  Without merge_cta it is also the     */
                                   /* state ring's size, which must fit in shared memory    */
    int64_t timeout_ns;            /* 0 = 2 s; bound on every device-side wait              */
    int32_t debug_flags;           /* 0; bit 0 makes the stop decision wait on a barrier    */
                                   /* nothing arrives on (exercises the bounded wait)       */
    art_launch_info_t *info;       /* host pointer or NULL                                  */
    int32_t prefetch;              /* 0 or -1 off, else 1..64 blocks pulled into L2         */
                                   /* ahead of the staged loads.  Pages read past the stop  */
                                   /* stay below window + prefetch blocks.                  */
    int32_t detector_off;          /* 0; 1 runs the walk without the ART detector: no      */
                                   /* statistic, no patience rule, every block consumed     */
                                   /* (stop_block = N_b).  The output equals the eps = 0    */
                                   /* walk's bit for bit.  A timing reference for the cost  */
                                   /* of the detector (the explainer's section 4 reports    */
                                   /* it with termination disabled); thresholds, P and      */
                                   /* min_blocks are ignored.  Built for BF16 caches on the */
                                   /* tensor-core engine with d = 128 and 64-token pages,   */
                                   /* and for F32 caches with d = 64, 16-token pages and    */
                                   /* at most 4 query heads per kv head; other cases return */
                                   /* ART_ERR_UNSUPPORTED, as does art_decode_attention_multi*/
                                   /* with n_queries = 2.                                   */
    int32_t merge_cta;             /* 0 auto; 1: the first CTA of each cluster only merges  */
                                   /* (its whole shared memory holds the block states, so   */
                                   /* the window can reach 64; its warps fold in parallel   */
                                   /* and one warp decides a batch behind them) while the   */
                                   /* others fetch and compute; -1 never.  Auto picks it    */
                                   /* for fewer units than SMs with clusters of 4 or more   */
                                   /* CTAs.  Built for BF16 caches on the tensor-core       */
                                   /* engine, d = 128, 64-token pages, single-query walks;  */
                                   /* 1 elsewhere returns ART_ERR_UNSUPPORTED, and with     */
                                   /* cluster_size 1 ART_ERR_PARAM.  Stops and outputs are  */
                                   /* the sequential rule's, as with every launch shape.    */
                                   /* 2: the same merge, reached through the workspace      */
                                   /* below instead of a cluster, so that more CTAs serve   */
                                   /* each unit (one merge CTA and W fetching CTAs per      */
                                   /* unit, all resident at once: a cooperative launch).    */
                                   /* Only on request; 2 without a workspace returns        */
                                   /* ART_ERR_NULL, with one too small ART_ERR_SHAPE.       */
    void *workspace;               /* device memory or NULL: scratch for merge_cta = 2      */
                                   /* (block states, ready tags and counters; at least      */
                                   /* art_workspace_bytes(p) bytes, 256-byte aligned).  It  */
                                   /* needs no clearing: every word is tagged with the      */
                                   /* call (a 32-bit count of this process's calls, so a    */
                                   /* word left untouched for 2^32 calls could read as      */
                                   /* current: clear a workspace idle that long before      */
                                   /* reuse).  Calls that overlap on the GPU must not share */
                                   /* one workspace.                                        */
    int64_t workspace_bytes;       /* its size                                              */
} art_params_t;

/*
 * art_decode_attention_ex -- the same step with per-sequence thresholds,
 * an explicit softmax scale, fetch accounting, device status, and launch
 * overrides.  Passing zeros for every option reproduces art_decode_attention.
 */
art_status_t art_decode_attention_ex(const art_params_t *p, art_stream_t stream);

/*
 * art_workspace_bytes -- the workspace art_decode_attention_ex can use for
 * this problem with merge_cta = 2: the tensors, options and
 * current device of p decide it.  Returns 0 when that walk does not apply
 * (more units than SMs, a cache type, head dim or page size it is not built
 * for, several query tokens), a negative art_status_t when the arguments are
 * invalid.  Nothing is launched.
 */
int64_t art_workspace_bytes(const art_params_t *p);

/*
 * art_decode_attention_no_alloc -- art_decode_attention_ex with merge_cta = 2
 * (one merge CTA and several fetching CTAs per unit, the block states handed
 * over through scratch memory), but the scratch is a fixed device array inside
 * this library, so the call allocates nothing.  The paper has no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc: a serving
 * engine whose memory pool has already claimed nearly all device memory (a
 * cudaMalloc there fails or steals from the pool), a latency-bound decode loop
 * that may not stall on an allocation (cudaMalloc and cudaFree can block the
 * host and synchronise the device), or a plug-in that may not grow the device
 * footprint of the application hosting it.
 *
 *  p           as for art_decode_attention_ex, except: workspace NULL and
 *              workspace_bytes 0 (else ART_ERR_PARAM), merge_cta 0 or 2
 *              (else ART_ERR_PARAM).  The caller still owns and passes every
 *              input and output tensor.
 *  Returns     ART_ERR_SCRATCH_SIZE when the problem needs more scratch than
 *              ART_NO_ALLOC_SCRATCH_BYTES even with the smallest ring (16
 *              block states per unit; about 67 KB per unit with 8 query heads
 *              per kv head, so about 60 units), ART_ERR_UNSUPPORTED where the
 *              workspace walk is not built (BF16 caches on the tensor-core
 *              engine, d = 128, 64-token pages, one query token, every CTA
 *              resident at once), otherwise what art_decode_attention_ex
 *              returns.  The ring is the largest that fits the array.
 *
 * The array (ART_NO_ALLOC_SCRATCH_BYTES, 256-byte aligned) is held by every
 * GPU on which the library's device code is loaded, until the process exits.
 * The first call on each device looks up the array's device address with that
 * device current and keeps it; make that first call before any stream capture
 * begins.  Every call on a device shares the one array and it keeps what the
 * last call left; nothing in it needs clearing, since each control word the
 * walk reads is tagged with the call that wrote it (a 32-bit count of the
 * process's calls: a word no call has rewritten for 2^32 calls could read as
 * current, which needs problems whose units shrink and then grow again across
 * that many calls).  Calls whose kernels
 * overlap on the GPU (other streams, other host threads) race on the array:
 * order them on one stream or serialise them.
 */
#define ART_NO_ALLOC_SCRATCH_BYTES (4 << 20)
art_status_t art_decode_attention_no_alloc(const art_params_t *p, art_stream_t stream);

/*
 * art_decode_attention_multi -- n_queries query tokens of each sequence (for
 * example draft tokens being verified together) share one walk of its cache:
 * every block is fetched once for all of them.  This is the decode form of
 * the cross-query reuse of shared KV entries in "QUILT: Rethinking
 * Sparse-Attention Prefill through Shared Query Execution" (Abstract); the
 * ART pages themselves only walk one query.
 *
 * Result: token t of sequence b gets exactly what art_decode_attention_ex
 * gives for q[b, t] alone -- its own statistics over its Hq/Hkv heads, its
 * own patience counter and stop, its output at its own stop.  The walk of a
 * (sequence, kv-head) ends when every token has stopped, so the blocks read
 * are those up to the latest token's stop, instead of each token reading its
 * own prefix.  All tokens of a sequence use the same order, page table,
 * thresholds and min_blocks.
 *
 * Tensors in p (everything else as in art_decode_attention_ex):
 *  q           [B, n_queries, Hq, d]   F32 or BF16; d contiguous; the token and
 *                                      head strides multiples of 16 bytes.
 *  out         [B, n_queries, Hq, d]   F32.
 *  stop_block  [B, n_queries, Hkv]     I32: blocks consumed by each token.
 * p->blocks_fetched counts the pages read by the shared walk of each unit.
 * Supported: n_queries = 1 (the single-query walk, on [B, 1, ...] tensors;
 * any size art_decode_attention_ex takes) or 2; with 2, d = 128 and
 * 2 * Hq/Hkv <= 8 (both tokens' heads fit the eight rows of one unit); BF16
 * on the tensor-core engine (engine 0 or 2), F32 on the CUDA-core engine.
 * Other cases return ART_ERR_UNSUPPORTED.
 * Errors as in art_decode_attention_ex; the library allocates nothing.
 */
art_status_t art_decode_attention_multi(const art_params_t *p, int32_t n_queries, art_stream_t stream);

/*
 * art_build_order_sink_recency -- write the default walk order: for each
 * sequence b with N_b = ceil(seq_lens[b] / page) blocks, block_order[b] =
 * [0, N_b-1, N_b-2, ..., 1] followed by -1 up to max_blocks (the sink block
 * first, then newest to oldest: section 2.4's "recency-first" traversal with
 * the mandatory block 0).  seq_lens: [B] I32; block_order: [B, max_blocks] I32
 * with a contiguous last dimension.  A sequence longer than max_blocks pages
 * gets only its first max_blocks entries (the attention call then reports it).
 */
art_status_t art_build_order_sink_recency(const art_tensor_t *seq_lens, int32_t page,
                                          art_tensor_t *block_order, art_stream_t stream);

/*
 * Importance-first traversal (section 2.4 names "importance-first" next to
 * "recency-first" as an order ART can run over, with block 0 kept first; the
 * explainer gives no importance estimate, so the one below is this
 * library's own).  Two calls:
 *
 * art_page_summary -- the summary of every page a sequence references: the
 * mean of the page's valid keys, per kv-head,
 *     summary[p, h, :] = (1/n) sum_{t < n} k_cache[p, h, t, :],
 * where p = page_table[b, j] for j < N_b and n = min(page, seq_lens[b] -
 * j*page).  Sums are fp32; the mean is rounded once to the summary's
 * type.  It reads the whole referenced K cache once: call it when
 * pages are filled (a page whose tokens do not change keeps its summary),
 * not per decode step.
 *   k_cache    [num_pages, Hkv, page, d] F32|BF16, d contiguous, 16-byte
 *              aligned base and strides (the layout art_decode_attention
 *              takes); d a power of two from 16 to 256.
 *   page_table [B, max_blocks] I32, seq_lens [B] I32 (as for the walk).
 *   summary    [num_pages, Hkv, d] F32|BF16 out, d contiguous, 16-byte
 *              aligned base and strides.  Pages no sequence references are
 *              not written.  A page referenced by several sequences must
 *              hold the same number of valid tokens in each.
 *   device_status  device [1] or NULL: a page-table entry outside
 *              [0, num_pages), or N_b > max_blocks, stores ART_ERR_BAD_INDEX
 *              there; the bad page is skipped.
 *
 * art_build_order_importance -- scores every block and writes the walk order
 * block 0 first, then blocks 1..N_b-1 by decreasing score, equal scores
 * newest (larger index) first, then -1 up to max_blocks.  The score of
 * block j of sequence b is the page mean of the attention logit summed over
 * all query heads (query head i reads kv-head i / G):
 *     block_scores[b, j] = sm_scale * sum_i q[b, i, :] . summary[page_table[b, j], i / G, :]
 * (fp32; -0 is stored as +0; -inf for j >= N_b).  The order is the exact
 * sort of the stored fp32 scores, so it is a permutation of 0..N_b-1 for any
 * input, NaN scores included, and is bitwise reproducible.
 *   q            [B, Hq, d] F32|BF16, d contiguous, 16-byte aligned base and
 *                strides; Hq a multiple of Hkv; Hkv*d at most 16384.
 *   summary      as written by art_page_summary (F32|BF16).
 *   page_table   [B, max_blocks] I32; seq_lens [B] I32; page > 0.
 *   sm_scale     the logit scale; <= 0 selects 1/sqrt(d).
 *   block_scores [B, max_blocks] F32 out, last dimension contiguous.
 *   block_order  [B, max_blocks] I32 out, last dimension contiguous; feed it
 *                to art_decode_attention.
 *   device_status  as above (bad page entries get a NaN score).
 * Both calls are asynchronous on the stream and allocate nothing.
 */
art_status_t art_page_summary(const art_tensor_t *k_cache, const art_tensor_t *page_table,
                              const art_tensor_t *seq_lens, art_tensor_t *summary,
                              int32_t *device_status, art_stream_t stream);

art_status_t art_build_order_importance(const art_tensor_t *q, const art_tensor_t *summary,
                                        const art_tensor_t *page_table, const art_tensor_t *seq_lens,
                                        int32_t page, float sm_scale, art_tensor_t *block_scores,
                                        art_tensor_t *block_order, int32_t *device_status,
                                        art_stream_t stream);

/* Static description of a status code. */
const char *art_strerror(art_status_t status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t art_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ART_H */
