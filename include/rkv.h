/*
 * rkv.h -- C ABI of the B200 (sm_100a) R-KV decode-time KV-cache compression step.
 *
 * R-KV ("R-KV: Redundancy-aware KV Cache Compression for Reasoning Models")
 * compresses a reasoning model's KV cache while it decodes.  Each time a
 * sequence's buffer of new tokens fills (every divide_length = 128 tokens),
 * for every layer and KV head, the step scores the cached tokens, keeps the
 * best budget - window of them plus the protected recent window, and
 * physically compacts K and V.  Sources (web pages about R-KV):
 *   [hysenlabs]   "R-KV: decoding-time KV cache compression for reasoning
 *                 models", sections "What the redundancy scoring actually
 *                 does at decode time", "Three install paths ...", "How this
 *                 differs from attention-sink and heavy-hitter eviction";
 *   [sourcepulse] R-KV project summary, section "How It Works";
 *   [atlas]       "R-KV: Redundancy-aware KV Cache Compression for Reasoning
 *                 Models" (atlas.scime.ai summary), sections "Approach" and
 *                 "Measured effects reported in the paper".
 *
 * Conventions for every entry point:
 *  - Pointers named k, v, q, I, R, r, Z, kept, cur_len, budgets, lambdas and
 *    workspace are DEVICE pointers; k_layers / v_layers / q_layers are HOST
 *    arrays holding device pointers.  The caller owns every buffer; the
 *    library allocates nothing, never synchronises the stream and keeps no
 *    state between calls.  Work is enqueued on `stream` (NULL = the legacy
 *    default stream) and can be captured in a CUDA graph.
 *  - bf16 tensors are raw 16-bit bfloat16 bit patterns (rkv_bf16).
 *  - K and V caches are [batch, n_kv_heads, cap, head_dim] per layer: row i of
 *    head h of sequence b starts at element ((b * n_kv_heads + h) * cap + i) *
 *    head_dim.  Q windows are [batch, n_q_heads, window, head_dim] per layer,
 *    the last `window` query vectors of every query head (rotary embedding
 *    already applied).  Query head g belongs to KV head g / G with
 *    G = n_q_heads / n_kv_heads.
 *  - Arguments are validated on the host before anything is enqueued; a bad
 *    argument returns an error status and enqueues nothing.  Faults found on
 *    the device (a sequence with an invalid budget, an out-of-range kept
 *    index, a bounded wait that ran out) set a flag in the workspace, which
 *    rkv_workspace_status() reads back.  No exception crosses this ABI.
 *  - Supported: head_dim == 128; 1 <= window <= budget; n_q_heads a multiple
 *    of n_kv_heads with G * window <= 64; device pointers 16-byte aligned.
 */
#ifndef RKV_H
#define RKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RKV_API __attribute__((visibility("default")))
#else
#define RKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t rkv_bf16;                  /* raw bfloat16 bits */
typedef struct CUstream_st *rkv_stream_t;   /* a cudaStream_t */
typedef struct CUevent_st *rkv_event_t;     /* a cudaEvent_t */

typedef enum {
    RKV_OK = 0,
    RKV_STATUS_DISABLED = 1,        /* budget <= 0 or buffer <= 0: compression off, nothing done */
    RKV_ERR_NULL = -1,              /* a required pointer is NULL */
    RKV_ERR_INVALID = -2,           /* inconsistent sizes (window, budget, cap, heads, lambda) */
    RKV_ERR_ALIGN = -3,             /* a device pointer or stride is not 16-byte aligned */
    RKV_ERR_ALIAS = -4,             /* outputs overlap inputs in a way the call does not allow */
    RKV_ERR_WORKSPACE = -5,         /* workspace NULL or smaller than rkv_workspace_size() */
    RKV_ERR_UNSUPPORTED = -6,       /* head_dim != 128, G * window > 64, cap too large, ... */
    RKV_ERR_CUDA = -7,              /* a CUDA runtime call or kernel launch failed */
    RKV_STATUS_DEVICE_TIMEOUT = -8, /* a bounded device-side wait ran out (read back later) */
    RKV_ERR_DEVICE_INPUT = -9       /* a device-side input was invalid (read back later) */
} rkv_status;

typedef enum {
    RKV_RED_MEAN = 0, /* r_i = mean cosine similarity to the other N-1 cached keys (default) */
    RKV_RED_MAX = 1   /* r_i = max cosine similarity to any other cached key */
} rkv_redundancy_mode;

typedef enum {
    RKV_GQA_MAX = 0, /* max over the query heads of a KV group (R-KV's choice, [atlas] table) */
    RKV_GQA_MEAN = 1 /* mean over the group: the ablation the table reports as worse */
} rkv_gqa_pool;

/* The knobs of the R-KV step ([hysenlabs] decode-time section and the
 * run_math.py flags in "Three install paths": kv_budget, window_size,
 * mix_lambda, divide_length). */
typedef struct {
    int32_t budget;          /* kv_budget: tokens kept per (sequence, layer, KV head) */
    int32_t buffer;          /* divide_length: new tokens between two compressions */
    int32_t window;          /* window_size: most recent tokens, never evicted */
    int32_t head_dim;        /* D; must be 128 */
    int32_t n_kv_heads;      /* Hkv */
    int32_t n_q_heads;       /* Hq, a multiple of Hkv */
    float mix_lambda;        /* lambda in Z = lambda I - (1 - lambda) R, finite */
    int32_t redundancy_mode; /* rkv_redundancy_mode */
    int32_t gqa_pool;        /* rkv_gqa_pool */
} rkv_config;

/* Optional extras of rkv_compress_step (pass NULL for none). */
typedef struct {
    int32_t *kept_out;       /* device [n_layers][batch][Hkv][cap] int32: for every compressed
                                unit, entries 0..budget-1 get the kept source indices in
                                ascending order; other entries are left untouched */
    float *scores_out;       /* device [n_layers][batch][Hkv][4][cap] fp32: I, r, R, Z of the
                                first N - window candidates of every compressed unit */
    rkv_event_t main_begin;  /* if not NULL: recorded on `stream` just before the main kernel */
    rkv_event_t main_end;    /* if not NULL: recorded on `stream` just after the main kernel */
    int32_t cluster_size;    /* CTAs per unit: 0 = automatic, 1 = one CTA per unit (K
                                streamed twice through shared memory), else a cluster of
                                2, 4, 8 or 16 CTAs that holds the unit's K on chip */
    rkv_event_t sim_begin;   /* MAX redundancy, if not NULL: recorded on `stream` just before
                                the first launch of the similarity kernel */
    rkv_event_t sim_end;     /* MAX redundancy, if not NULL: recorded just after its last */
} rkv_step_options;

/* Human-readable name of a status code (static storage). */
RKV_API const char *rkv_status_string(rkv_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
RKV_API int32_t rkv_version(void);

/* The CUDA runtime error code (a cudaError_t value) behind the most recent
 * RKV_ERR_CUDA that a call of this library returned on the calling thread, or 0
 * when there was none.  Host-only; it does not touch the device. */
RKV_API int32_t rkv_last_cuda_error(void);

/*
 * Bytes of device workspace every call below needs for the given shapes
 * (n_layers = batch = 1 and cap = the per-head row count for the per-head
 * entry points).  Returns 0 for an invalid config.  The workspace needs
 * 256-byte alignment, holds no state between calls and may be reused.  The
 * size includes room for one int32 per sequence in which the batched steps
 * order the sequences by decreasing length, so that their units start with the
 * longest; a workspace short of exactly that room (256-byte rounded) is still
 * accepted, and the units then run in launch order (the results are the same).
 */
RKV_API size_t rkv_workspace_size(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap);

/*
 * Reads the device-side status word of a workspace used by earlier calls on
 * `stream`: synchronises the stream, then returns RKV_OK,
 * RKV_STATUS_DEVICE_TIMEOUT or RKV_ERR_DEVICE_INPUT.  Every call resets the
 * word at its start, so this reports on the latest call only.
 */
RKV_API rkv_status rkv_workspace_status(const void *workspace, rkv_stream_t stream);

/*
 * The launch shape rkv_compress_step picks (cluster_size = 0) for n_units
 * (sequence, layer, KV head) units in one call (n_layers * batch * n_kv_heads)
 * with caches of `cap` rows: CTAs per unit (1: one CTA per unit, the choice
 * once the call has at least one unit per SM; else the cluster size), rows
 * each CTA owns, and dynamic shared memory per CTA.  Host-only (no CUDA
 * call).  RKV_ERR_UNSUPPORTED when no shape fits; any output pointer may be
 * NULL.
 */
RKV_API rkv_status rkv_query_step_shape(const rkv_config *cfg, int64_t n_units, int32_t cap,
                                        int32_t *cluster_size, int32_t *rows_per_cta,
                                        size_t *smem_bytes);

/*
 * Importance I for one (sequence, layer): step 1 of R-KV ("importance
 * (derived from attention weights)", [sourcepulse] How It Works; max pooling
 * over the GQA group, [atlas] Measured effects table).
 *   s_{g,j,i} = q_{g,j} . k_i / sqrt(D), query j of the window sitting at
 *   position M + j and seeing keys 0..M+j; softmax over i; mean over the
 *   window queries j; max (or mean, cfg->gqa_pool) over the G query heads of
 *   the group; restricted to the M = n_tokens - window candidates and
 *   renormalised to sum 1.
 * q: [Hq][window][128]; k: head h, row i at k + h * k_head_stride + i * 128
 * (k_head_stride a multiple of 128, >= n_tokens * 128); window < n_tokens.
 * I: [Hkv][M] fp32 out.  inv_norm: [Hkv][n_tokens] fp32 out, 1/max(||k_i||, 1e-12),
 * or NULL.
 */
RKV_API rkv_status rkv_score_importance(const rkv_config *cfg, const rkv_bf16 *q, const rkv_bf16 *k,
                                int64_t k_head_stride, int32_t n_tokens, float *I,
                                float *inv_norm, void *workspace, size_t ws_bytes,
                                rkv_stream_t stream);

/*
 * Redundancy for one (sequence, layer): step 2 of R-KV ("redundancy
 * (key-vector cosine similarity)", [atlas] summary and Approach; near
 * duplicates found by cosine similarity, [sourcepulse] How It Works).
 *   c_ij = khat_i . khat_j with khat = k / max(||k||, 1e-12);
 *   MEAN: r_i = sum_{j < N, j != i} c_ij / (N - 1);  MAX: r_i = max_{j < N, j != i} c_ij;
 *   R = softmax over the M candidates of r.
 * k as in rkv_score_importance.  r, R: [Hkv][M] fp32 out (either may be NULL).
 */
RKV_API rkv_status rkv_score_redundancy(const rkv_config *cfg, const rkv_bf16 *k, int64_t k_head_stride,
                                int32_t n_tokens, float *r, float *R, void *workspace,
                                size_t ws_bytes, rkv_stream_t stream);

/*
 * Joint score and selection for one (sequence, layer): steps 3-4 of R-KV
 * (Z = lambda I - (1 - lambda) R, [atlas] Approach; top-k within the budget,
 * [sourcepulse] How It Works; protected recent window, [hysenlabs]).
 * I, R: [Hkv][M] fp32 in, M = n_tokens - window.  Keeps the budget - window
 * candidates with the largest Z (ties: lower index first) and the window
 * M..n_tokens-1.  kept: [Hkv][budget] int32 out, ascending.  Z: [Hkv][M] fp32
 * out or NULL.
 */
RKV_API rkv_status rkv_select_topk(const rkv_config *cfg, const float *I, const float *R,
                           int32_t n_tokens, int32_t *kept, float *Z, void *workspace,
                           size_t ws_bytes, rkv_stream_t stream);

/*
 * Physical compaction for one (sequence, layer): step 5 of R-KV (eviction,
 * not masking, [hysenlabs] "How this differs ..."; the SGLang port's
 * two-phase compaction in the decode-time section).
 * For every head h and t < budget: k_dst[h][t] = k_src[h][kept[h][t]] and the
 * same for V, bit for bit.  kept: [Hkv][budget], every entry in
 * [0, n_tokens).  head_stride (elements) applies to all four tensors.
 * k_dst == k_src and v_dst == v_src compacts in place (all of a head's source
 * rows are read before any of its rows is written); otherwise the
 * destinations must not overlap any source (RKV_ERR_ALIAS).
 */
RKV_API rkv_status rkv_compact_kv(const rkv_config *cfg, const rkv_bf16 *k_src, const rkv_bf16 *v_src,
                          const int32_t *kept, rkv_bf16 *k_dst, rkv_bf16 *v_dst,
                          int64_t head_stride, int32_t n_tokens, void *workspace,
                          size_t ws_bytes, rkv_stream_t stream);

/*
 * The whole R-KV step over a batch of sequences and all layers, in place
 * ("applied periodically during decoding with a fixed buffer", [atlas]
 * Approach; compression only when budget and buffer are both positive,
 * [hysenlabs] "Three install paths").
 *   For every sequence b with budget_b > 0, buffer > 0 and
 *   cur_len[b] >= budget_b + buffer ("due"), for every layer and KV head:
 *   steps 1-5 above over its N = cur_len[b] cached tokens; then
 *   cur_len[b] = budget_b.  Sequences that are not due are left untouched.
 * k_layers, v_layers: host arrays [n_layers] of device pointers to
 *   [batch][Hkv][cap][128] bf16 caches (updated in place);
 * q_layers: host array [n_layers] of device pointers to [batch][Hq][window][128];
 * budgets: device [batch] int32, or NULL for cfg->budget;
 * lambdas: device [batch] fp32, or NULL for cfg->mix_lambda;
 * cur_len: device [batch] int32, read and updated.
 * Returns RKV_STATUS_DISABLED (nothing enqueued) when cfg->budget <= 0 or
 * cfg->buffer <= 0 and no per-sequence budgets are given.
 */
RKV_API rkv_status rkv_compress_step(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                             int32_t cap, rkv_bf16 *const *k_layers, rkv_bf16 *const *v_layers,
                             const rkv_bf16 *const *q_layers, const int32_t *budgets,
                             const float *lambdas, int32_t *cur_len,
                             const rkv_step_options *opts, void *workspace, size_t ws_bytes,
                             rkv_stream_t stream);

/*
 * The decode side of the loop: appends n_new tokens' keys and values to every
 * sequence's cache at its current length, then cur_len[b] += n_new.  Together
 * with rkv_compress_step this is the decode-time cycle of R-KV: tokens
 * accumulate in the buffer until it holds divide_length = buffer new tokens,
 * then the step compresses back to the budget ("applied periodically during
 * decoding with a fixed buffer", [atlas] Approach).
 * k_new_layers / v_new_layers: host arrays [n_layers] of device pointers to
 * [batch][Hkv][n_new][128] bf16; k_layers / v_layers, cap and cur_len as in
 * rkv_compress_step.  A sequence without room for n_new more rows is left
 * untouched and reported through the workspace status (RKV_ERR_DEVICE_INPUT).
 */
RKV_API rkv_status rkv_append_kv(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                 int32_t cap, rkv_bf16 *const *k_layers,
                                 rkv_bf16 *const *v_layers,
                                 const rkv_bf16 *const *k_new_layers,
                                 const rkv_bf16 *const *v_new_layers, int32_t n_new,
                                 int32_t *cur_len, void *workspace, size_t ws_bytes,
                                 rkv_stream_t stream);

/*
 * The whole step as rkv_compress_step, for callers that cannot allocate
 * device memory, so cannot hand over a workspace.  Examples are a plugin
 * inside a serving engine that owns all of the GPU's memory, or a decode loop
 * where an allocation (which may synchronise the device) is not allowed.  The
 * R-KV pages have no counterpart: this is a packaging variant, not part of
 * the method.
 *
 * Instead of a workspace the call uses a fixed scratch array of
 * RKV_NOALLOC_SCRATCH_BYTES in the library's own device memory.  It holds a
 * status header and one int32 per sequence, so batch is limited to
 * RKV_NOALLOC_MAX_BATCH; a larger batch returns RKV_ERR_UNSUPPORTED.  Only
 * MEAN redundancy fits: MAX keeps r of every (layer, sequence, head) in the
 * workspace, so redundancy_mode RKV_RED_MAX returns RKV_ERR_UNSUPPORTED.
 * Every GPU on which the library is used keeps this array until the process
 * exits.
 *
 * The first call on each device (or of rkv_noalloc_status) looks up the
 * array's device address with cudaGetSymbolAddress, with that device current,
 * and caches it for the life of the process; make that first call before any
 * stream capture, and do not use these two calls after cudaDeviceReset (the
 * cached address would be stale).  The call allocates nothing (no cudaMalloc,
 * no cudaFree, no allocating library routine).  All calls share the one array
 * and it keeps whatever the last call left in it; the call resets what must
 * start at zero itself.  Calls whose work overlaps on the GPU (two streams,
 * two host threads) race on the array: serialise them.  Other arguments,
 * results and host-side statuses are those of rkv_compress_step; faults found
 * on the device land in the array's status word, which rkv_noalloc_status
 * reads back.
 */
#define RKV_NOALLOC_MAX_BATCH 4096
#define RKV_NOALLOC_SCRATCH_BYTES (256 + 4 * RKV_NOALLOC_MAX_BATCH)
RKV_API rkv_status rkv_compress_step_noalloc(const rkv_config *cfg, int32_t n_layers,
                                             int32_t batch, int32_t cap,
                                             rkv_bf16 *const *k_layers,
                                             rkv_bf16 *const *v_layers,
                                             const rkv_bf16 *const *q_layers,
                                             const int32_t *budgets, const float *lambdas,
                                             int32_t *cur_len, const rkv_step_options *opts,
                                             rkv_stream_t stream);

/*
 * The device-side status of the latest rkv_compress_step_noalloc call on the
 * current device, as rkv_workspace_status reports it for a workspace:
 * synchronises `stream`, then returns RKV_OK, RKV_STATUS_DEVICE_TIMEOUT or
 * RKV_ERR_DEVICE_INPUT (for instance a sequence whose per-sequence budget is
 * below the window, which the step skipped).  No counterpart in the R-KV
 * pages either.
 */
RKV_API rkv_status rkv_noalloc_status(rkv_stream_t stream);

/*
 * Shared selection: every KV head of a (sequence, layer) keeps the same
 * tokens, and with the heads split over tensor-parallel ranks every rank
 * evicts the identical set (hysenlabs write-up, decode-time section: the vLLM
 * port's cross-rank eviction-score all-reduce; "every TP rank evicts the
 * identical set").  The score of candidate i is the sum over all KV heads of
 * the per-head joint scores, Zsum_i = sum_h Z_h[i]; the kept set is the top
 * budget - window candidates of Zsum by (score desc, index asc) plus the
 * window.  Two calls around the caller's all-reduce:
 *
 *   rkv_score_shared            per-head Z of this call's KV heads, summed
 *                               over them into z_sum (the rank's part)
 *   (caller)                    all-reduce (sum) of z_sum over the ranks
 *   rkv_select_compact_shared   one select per (sequence, layer) on the
 *                               complete z_sum; every head of this call is
 *                               compacted in place with that set
 *
 * Arguments as rkv_compress_step; n_kv_heads / n_q_heads are this rank's
 * heads.  z_sum: device [n_layers][batch][cap] fp32, 16-byte aligned; every
 * entry is written (0 past the candidates and for sequences that are not
 * due), so ranks reduce defined data.  Due sequences are those with
 * cur_len >= budget + buffer; rkv_score_shared leaves cur_len unchanged and
 * rkv_select_compact_shared sets it to the budget.  kept_out (optional):
 * device [n_layers][batch][cap] int32, entries 0..budget-1 of every compressed
 * (layer, sequence) get the kept rows in ascending order.  Both calls use one
 * workspace of rkv_workspace_size_shared bytes (which also carries the
 * per-head scores from the first call to nothing but itself; the second call
 * needs only z_sum).  Caches up to about 6700 rows (one CTA per head);
 * longer caches: RKV_ERR_UNSUPPORTED.
 */
RKV_API size_t rkv_workspace_size_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                         int32_t cap);

RKV_API rkv_status rkv_score_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                    int32_t cap, const rkv_bf16 *const *k_layers,
                                    const rkv_bf16 *const *q_layers, const int32_t *budgets,
                                    const float *lambdas, const int32_t *cur_len, float *z_sum,
                                    void *workspace, size_t ws_bytes, rkv_stream_t stream);

RKV_API rkv_status rkv_select_compact_shared(const rkv_config *cfg, int32_t n_layers,
                                             int32_t batch, int32_t cap, rkv_bf16 *const *k_layers,
                                             rkv_bf16 *const *v_layers, const int32_t *budgets,
                                             int32_t *cur_len, const float *z_sum,
                                             int32_t *kept_out, void *workspace, size_t ws_bytes,
                                             rkv_stream_t stream);

/*
 * Paged caches: each layer's keys and values
 * live in page pools [num_pages][Hkv][page_rows][128] bf16, and sequence b
 * owns the pages block_table[b][0..] in logical order (logical row i of a
 * sequence is slot i % page_rows of page block_table[b][i / page_rows]; the
 * table is shared by all layers).  The step is rkv_compress_step's, reading
 * and compacting rows through the table; afterwards the pages a compressed
 * sequence no longer needs, ceil(budget / P) .. ceil(N / P) - 1, are listed
 * for the caller's allocator: physical eviction that returns freed blocks
 * (hysenlabs write-up, decode-time section: the FREE_BLOCKS return path).
 */
typedef struct {
    const int32_t *block_table; /* device [batch][max_blocks] page ids */
    int32_t max_blocks;         /* row stride of block_table; max_blocks * page_rows = cap */
    int32_t page_rows;          /* P: 16, 32, 64 or 128 */
    int32_t num_pages;          /* pages in each layer's pool */
    int32_t *freed_pages;       /* device [batch][max_blocks]: entries 0..n_freed[b]-1 get the
                                   page ids sequence b gave back (in logical order) */
    int32_t *n_freed;           /* device [batch]: pages given back (0 when not compressed) */
} rkv_paged_kv;

/*
 * The step on paged caches.  k_pools / v_pools: host arrays [n_layers] of
 * device pointers to the page pools; q_layers, budgets, lambdas, cur_len,
 * opts (kept_out / scores_out / events; cluster_size 0 or 1) and the
 * workspace (rkv_workspace_size with cap = max_blocks * page_rows) as in
 * rkv_compress_step (MAX redundancy reads its similarity tiles through the
 * block table too); pages of different sequences must be distinct.  Caches up to 512 pages per
 * sequence and one CTA's rows (rkv_query_step_shape cluster_size 1).
 */
RKV_API rkv_status rkv_compress_step_paged(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                           const rkv_paged_kv *pg, rkv_bf16 *const *k_pools,
                                           rkv_bf16 *const *v_pools,
                                           const rkv_bf16 *const *q_layers,
                                           const int32_t *budgets, const float *lambdas,
                                           int32_t *cur_len, const rkv_step_options *opts,
                                           void *workspace, size_t ws_bytes, rkv_stream_t stream);

/*
 * Caches with per-sequence capacities.  Each layer's keys live in one pool of
 * pool_rows rows of 128 bf16 (256 bytes), and so do its values (a second pool
 * of the same geometry).  Sequence b owns the block of n_kv_heads *
 * seq_cap[b] rows starting at row seq_row[b]: row i of KV head h of sequence
 * b is pool row seq_row[b] + h * seq_cap[b] + i.  This is the
 * [batch, kv_heads, len, head_dim] layout of rkv_compress_step with the batch
 * split into blocks of their own size, so a sequence with a small budget
 * holds budget + buffer rows instead of the largest sequence's (the pages'
 * fixed buffer per sequence: atlas.scime.ai summary, "Approach"; the 90%
 * memory saving: sourcepulse summary, "Highlighted Details").  Blocks of
 * different sequences must not overlap; gaps between them are allowed.
 */
typedef struct {
    const int64_t *seq_row;   /* device [batch]: first pool row of sequence b (8-byte aligned) */
    const int32_t *seq_cap;   /* device [batch]: rows per KV head of sequence b's block */
    int64_t pool_rows;        /* rows in each layer's pool (<= INT32_MAX) */
    int32_t max_cap;          /* an upper bound of every seq_cap[b]: sizes shared memory, the
                                 workspace (rkv_workspace_size with cap = max_cap) and the
                                 row stride of kept_out / scores_out */
} rkv_ragged_kv;

/*
 * The step on caches with per-sequence capacities (layout above): for every
 * due sequence (cur_len[b] >= budget_b + buffer), for every layer and KV head,
 * steps 1-5 over its N = cur_len[b] rows, then cur_len[b] = budget_b, exactly
 * as rkv_compress_step.  k_pools / v_pools: host arrays [n_layers] of device
 * pointers to the pools; q_layers, budgets, lambdas, cur_len as in
 * rkv_compress_step; opts: kept_out / scores_out as there with cap = max_cap,
 * events, cluster_size 0 or 1 (one CTA per unit; clusters:
 * RKV_ERR_UNSUPPORTED).  A due sequence whose block does not fit the pool
 * (seq_row[b] < 0, seq_row[b] + n_kv_heads * seq_cap[b] > pool_rows,
 * seq_cap[b] > max_cap) or whose cur_len exceeds seq_cap[b] is skipped and
 * reported through the workspace status (RKV_ERR_DEVICE_INPUT).
 */
RKV_API rkv_status rkv_compress_step_ragged(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                            const rkv_ragged_kv *rg, rkv_bf16 *const *k_pools,
                                            rkv_bf16 *const *v_pools,
                                            const rkv_bf16 *const *q_layers,
                                            const int32_t *budgets, const float *lambdas,
                                            int32_t *cur_len, const rkv_step_options *opts,
                                            void *workspace, size_t ws_bytes, rkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RKV_H */
