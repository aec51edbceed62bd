/*
 * kvc.h -- C ABI of libkvc: attention-guided KV-cache eviction and in-place paged
 * compaction on NVIDIA B200 (sm_100a).
 *
 * The path has five steps, each an entry point below:
 *   1. kvc_score_from_lse      score every cached entry by the attention it receives
 *                              from a query set, recovered from the attention
 *                              log-sum-exp ("ActKV Dissected", Component 3 and
 *                              Component 1; "BeaconKV", Key ideas, for beacon plus
 *                              recent queries)
 *   2. kvc_lrfu_update         fold the action-critical hit signal into an LRFU
 *                              combined recency-frequency value, lambda = 0.5
 *                              ("ActKV Dissected", Component 1)
 *   3. kvc_confidence_ratchet  top-20 average-NLL confidence monitor, min-pooled
 *                              (window 64, stride 8), linear-fit slope, one-way
 *                              x1.75 budget ratchet from 512 to 30,000
 *                              ("ActKV Dissected", Summary, Component 2, Lineage)
 *      kvc_select_budget       keep the top-budget entries per row, ties broken by
 *                              lower token position
 *   4. kvc_plan_slots          conflict-free slot plan: survivors outside the target
 *                              region paired one-to-one with holes inside it
 *                              ("ActKV Dissected", Component 3)
 *   5. kvc_compact_pages       one parallel in-place copy pass; shrunk block table
 *                              and freed-page list ("ActKV Dissected", Component 3)
 *
 * Next to the path, building its query set:
 *      kvc_beacon_update       beacon queries kept by online k-means over each
 *                              group's past queries ("BeaconKV", Key ideas)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer inside the structures and every array argument is DEVICE memory
 *   owned by the caller, unless stated otherwise.  The library never allocates,
 *   frees or synchronises; it keeps no state between calls except a thread-local
 *   last-error string.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 * - Errors the host can see (null pointers, unsupported dtype or head_dim, sizes)
 *   return a status other than KVC_OK before anything is enqueued.
 *   kvc_last_error() then describes the problem.
 * - Errors only the device can see (a page id outside the pool, a row length over
 *   capacity, a non-finite value, a full freed list, a wait that gave up) are
 *   written to `d_status` when it is not NULL: d_status points to two device
 *   int32 values {code, row}, which the caller zeroes; the first error wins and
 *   later ones are dropped.  The offending row is skipped; no kernel traps.  The
 *   caller reads d_status after synchronising.
 * - A "row" is one (sequence, layer, KV head) stream of cached entries:
 *       row = (seq * num_layers + layer) * num_kv_heads + kv_head.
 *   Its logical slots are 0 .. row_len[row]-1; slot i lives in physical page
 *   block_table[row][i / page_size] at offset i % page_size.
 * - Inputs are not modified except the arrays documented as in/out.
 * - Calls on disjoint buffers may run concurrently on different streams.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvc_stream_t; /* same type as cudaStream_t */

typedef enum {
    KVC_OK = 0,
    KVC_ERR_INVALID_ARGUMENT = 1, /* null pointer, size out of range, inconsistent shapes */
    KVC_ERR_UNSUPPORTED = 2,      /* valid but not implemented (dtype, head_dim, page_size) */
    KVC_ERR_CUDA = 3,             /* a CUDA runtime call failed (launch, attribute, tensor map) */
    KVC_ERR_DEVICE_FAULT = 4,     /* reserved for callers that fold d_status into a kvc_status */
    KVC_ERR_TIMEOUT = 5           /* reserved for callers that fold d_status into a kvc_status */
} kvc_status;

/* codes written to d_status[0] by kernels */
#define KVC_DEV_OK 0
#define KVC_DEV_BAD_PAGE 1       /* page id outside [0, num_pages), or -1 inside a row's length */
#define KVC_DEV_BAD_LENGTH 2     /* row_len < 0 or > max_pages_per_row * page_size, or new length > row_len */
#define KVC_DEV_NONFINITE 3      /* NaN or +inf in an LSE, score, CRF or logit */
#define KVC_DEV_KEPT_MISMATCH 4  /* kept[row] differs from the number of set bytes in keep */
#define KVC_DEV_FREED_OVERFLOW 5 /* freed list longer than freed_capacity */
#define KVC_DEV_BAD_MOVE 6       /* a move outside [0, row_len) or not hole/survivor */
#define KVC_DEV_TIMEOUT 7        /* a bounded wait inside a kernel gave up */
#define KVC_DEV_BAD_STEPS 8      /* step table not ascending from 0, num_steps out of range, or a negative position */

typedef enum { KVC_F32 = 0, KVC_BF16 = 1 } kvc_dtype;

/*
 * The paged cache (layout adopted for per-KV-head eviction: a page holds
 * page_size tokens of ONE (layer, KV head) row, so rows compact independently).
 *   k_pool, v_pool  [num_pages][page_size][head_dim] of `dtype`, same page ids;
 *                   16-byte aligned.  In/out for kvc_compact_pages only.
 *   block_table     [rows][max_pages_per_row] int32, -1 = no page.  In/out for compaction.
 *   row_len         [rows] int32.  In/out for compaction.
 *   slot_pos        [rows][max_pages_per_row * page_size] int32: the original token
 *                   position of each logical slot (order after compaction is not
 *                   position order).  In/out for compaction.
 *   slot_label      same shape, uint8: 0 observation, 1 reasoning, 2 action; may be
 *                   NULL.  In/out for compaction.
 */
typedef struct {
    void *k_pool;
    void *v_pool;
    int64_t num_pages;
    int32_t page_size;
    int32_t head_dim;
    int32_t dtype; /* kvc_dtype */
    int32_t max_pages_per_row;
    int32_t *block_table;
    int32_t *row_len;
    int32_t *slot_pos;
    uint8_t *slot_label;
    int32_t num_seqs;
    int32_t num_layers;
    int32_t num_kv_heads;
    int32_t reserved;
} kvc_cache;

/*
 * The query set of one round (action-region tokens, or beacon plus recent queries).
 *   q      [num_seqs][num_layers][max_q][num_q_heads][head_dim], the cache's dtype,
 *          16-byte aligned.  Query head h belongs to KV head h / (num_q_heads / num_kv_heads).
 *   lse    [num_seqs][num_layers][num_q_heads][max_q] fp32, natural log of the softmax
 *          denominator of each query column over the keys it attended to.  Input to
 *          scoring; output of kvc_query_lse.  -inf marks a column that saw no key.
 *   q_pos  [num_seqs][max_q] int32 token position of each query (causal mask: a query
 *          sees keys whose slot_pos <= q_pos); INT32_MAX marks an unmasked beacon.
 *   num_q  [num_seqs] int32 number of valid queries (the first num_q[seq] of max_q).
 */
typedef struct {
    const void *q;
    float *lse;
    const int32_t *q_pos;
    const int32_t *num_q;
    int32_t max_q;
    int32_t num_q_heads;
} kvc_queries;

/* flags of kvc_score_from_lse */
#define KVC_SCORE_ACCUMULATE 1u  /* add into scores instead of overwriting them */
#define KVC_SCORE_COMPUTE_LSE 2u /* run kvc_query_lse first (beacons have no decode-time LSE) */
#define KVC_SCORE_SIMT 4u        /* force the CUDA-core path even for bf16 (cross-check) */

/* flags of kvc_lrfu_update */
#define KVC_HIT_BINARY 1u /* a hit counts 1 instead of its attention score */

typedef struct {
    int32_t top_k;      /* tokens averaged per step: 20 */
    int32_t window;     /* min-pool window: 64 */
    int32_t stride;     /* min-pool stride: 8 */
    int32_t grow_num;   /* growth factor numerator: 7  (7/4 = 1.75) */
    int32_t grow_den;   /* growth factor denominator: 4 */
    int32_t init_budget;/* 512 */
    int32_t cap;        /* 30000 */
    int32_t min_points; /* pooled points needed before a fit: 2 */
    int32_t max_steps;  /* largest `steps` of one kvc_confidence_ratchet call (sizes the state) */
    int32_t reserved;
} kvc_ratchet_params;

/* Per-sequence ratchet state as laid out in the state buffer (documented so that a
 * caller can snapshot, restore or inspect it).  The buffer holds num_seqs of these,
 * then num_seqs histories of (window - 1 + max_steps) floats. */
typedef struct {
    int64_t steps_seen;       /* decode steps consumed so far */
    int64_t last_expand_step; /* steps_seen at the last expansion (0 before any) */
    int64_t next_window;      /* index of the first pooled window not yet emitted */
    double fit_n, fit_sx, fit_sy, fit_sxy, fit_sxx; /* OLS sums since the last expansion */
    double last_slope;        /* slope of the last evaluation, NaN when none was made */
    int32_t budget;
    int32_t expansions;
    int32_t last_points;      /* pooled points in the last fit */
    int32_t reserved;
} kvc_ratchet_seq_state;

const char *kvc_status_string(kvc_status status);
const char *kvc_last_error(void);
int32_t kvc_version(void);

/*
 * Step 1 (input of): natural-log LSE of every valid query column over the keys it
 * sees in its row (causal by slot_pos; beacons see all keys), written to queries->lse.
 * Stands in for the LSE a paged-attention kernel emits beside its output
 * ("ActKV Dissected", Component 3); needed for beacon queries, which no attention
 * produced ("BeaconKV", Key ideas).  Columns that see no key get -inf.
 */
kvc_status kvc_query_lse(const kvc_cache *cache, const kvc_queries *queries, int32_t *d_status,
                         kvc_stream_t stream);

/*
 * Step 1: scores[row][slot] = sum over valid queries j of the row's sequence and layer,
 * and over the query heads g of the row's GQA group, of
 *     [q_pos_j >= slot_pos] * exp(q_{j,g} . k_slot / sqrt(head_dim) - lse_{j,g}).
 * scores: [rows][max_pages_per_row * page_size] fp32, written for slots < row_len only.
 * bf16 caches run on the tensor cores (tcgen05, TMA page gather); fp32 caches on CUDA
 * cores in fp32.  Requires page_size 16 and head_dim 64 or 128 for bf16.
 */
kvc_status kvc_score_from_lse(const kvc_cache *cache, const kvc_queries *queries, float *scores,
                              uint32_t flags, int32_t *d_status, kvc_stream_t stream);

/*
 * Step 2: per row, the hit signal is the row's action-critical entries -- the shortest
 * prefix of the order (score descending, slot_pos ascending, slot ascending) whose mass
 * reaches hit_mass * (total score) -- and then
 *     crf[row][slot] <- h + 2^(-lambda * dt_rounds) * crf[row][slot]
 * with h = score (or 1 with KVC_HIT_BINARY) for hits and 0 otherwise.  hit_mass >= 1
 * turns the gate off (every entry with a positive score is a hit).  crf is in/out,
 * [rows][max_slots] fp32, updated for slots < row_len.
 */
kvc_status kvc_lrfu_update(const kvc_cache *cache, const float *scores, float *crf, float lambda,
                           float hit_mass, int32_t dt_rounds, uint32_t flags, int32_t *d_status,
                           kvc_stream_t stream);

/*
 * Step 3 (selection): keep[row][slot] = 1 for the first min(budget[seq], row_len) slots of
 * the order (crf descending, slot_pos ascending, slot ascending), 0 for the rest of the
 * row.  Entries whose label bit is set in protect_label_mask are always kept and use up
 * budget first.  kept[row] = number kept.  budget is [num_seqs] int32 on the device
 * (the ratchet's output).  keep: [rows][max_slots] uint8 (written for slots < row_len).
 */
kvc_status kvc_select_budget(const kvc_cache *cache, const float *crf, const int32_t *budget,
                             uint32_t protect_label_mask, uint8_t *keep, int32_t *kept,
                             int32_t *d_status, kvc_stream_t stream);

/*
 * Steps 2 and 3b in one launch: the same arguments, the same checks and the same results as
 * kvc_lrfu_update(cache, scores, crf, lambda, hit_mass, dt_rounds, flags, ...) followed by
 * kvc_select_budget(cache, crf, budget, protect_label_mask, keep, kept, ...) on one stream.
 * One cluster per row runs both: the selection reads the LRFU values the cluster has just
 * written, with no second launch.  (A system-level fusion of two steps of "ActKV Dissected",
 * Component 1 and Summary; the pages have no counterpart of the entry point itself.)
 */
kvc_status kvc_lrfu_select(const kvc_cache *cache, const float *scores, float *crf, float lambda, float hit_mass,
                           int32_t dt_rounds, uint32_t flags, const int32_t *budget, uint32_t protect_label_mask,
                           uint8_t *keep, int32_t *kept, int32_t *d_status, kvc_stream_t stream);

/*
 * Step 4: with m = kept[row], the holes are the slots i < m with keep 0 and the
 * survivors are the slots i >= m with keep 1, both ascending; move j copies survivor j
 * into hole j.  move_src/move_dst: [rows][max_slots] int32 (first num_moves[row] valid).
 * No slot is written twice and no destination is a source, so one parallel pass is safe.
 * A row whose kept count disagrees with its mask (as many holes before m as survivors
 * after it is the condition), or whose row_len is out of range, is reported in d_status
 * (KVC_DEV_KEPT_MISMATCH / KVC_DEV_BAD_LENGTH) and gets num_moves[row] = -1; the
 * compaction leaves such a row exactly as it is.
 */
kvc_status kvc_plan_slots(const kvc_cache *cache, const uint8_t *keep, const int32_t *kept,
                          int32_t *move_src, int32_t *move_dst, int32_t *num_moves,
                          int32_t *d_status, kvc_stream_t stream);

/*
 * kvc_select_budget followed by kvc_plan_slots, in one launch: the same arguments, checks,
 * device errors and results (keep, kept, move_src, move_dst, num_moves) as the two calls in
 * sequence, with the plan reading the keep mask and kept counts this launch has just written.
 * (A system-level fusion of two steps of "ActKV Dissected", Summary and Component 3; the pages
 * have no counterpart of the entry point itself.)
 */
kvc_status kvc_select_plan(const kvc_cache *cache, const float *crf, const int32_t *budget,
                           uint32_t protect_label_mask, uint8_t *keep, int32_t *kept,
                           int32_t *move_src, int32_t *move_dst, int32_t *num_moves,
                           int32_t *d_status, kvc_stream_t stream);

/* bytes of device workspace kvc_compact_pages needs for `rows` rows */
size_t kvc_compact_workspace_bytes(int32_t rows);

/*
 * Step 5: for every move, copy the K and V vectors and slot_pos, slot_label and (when
 * crf is not NULL) crf from the source slot to the destination slot, in place.  Then,
 * with m = new_len[row] (the kept count) and n = row_len[row]: the row's logical pages
 * ceil(m/P) .. ceil(n/P)-1 are appended to `freed` (rows in order, pages ascending
 * within a row) and set to -1 in the block table, and row_len[row] = m.
 * freed: [freed_capacity] int32; *num_freed (device int64) = total freed.  Source slots
 * are not cleared.  workspace: at least kvc_compact_workspace_bytes(rows) bytes of
 * device memory whose contents need not be preserved between calls.
 * A row is compacted only when 0 <= new_len <= row_len <= max_slots and
 * 0 <= num_moves <= min(new_len, row_len - new_len); any other row (num_moves = -1 from
 * the planner included) keeps its pool bytes, block table, positions and row_len.
 * Freed-list overflow (KVC_DEV_FREED_OVERFLOW): *num_freed is the total the list would
 * need, so it can exceed freed_capacity; the rows whose pages fit are listed as usual;
 * a row whose pages do not all fit lists none of them and keeps those block-table
 * entries (the pages stay mapped, unused), while its row_len is still set to new_len.
 */
kvc_status kvc_compact_pages(const kvc_cache *cache, const int32_t *move_src, const int32_t *move_dst,
                             const int32_t *num_moves, const int32_t *new_len, float *crf,
                             int32_t *freed, int64_t freed_capacity, int64_t *num_freed,
                             void *workspace, size_t workspace_bytes, int32_t *d_status,
                             kvc_stream_t stream);

/*
 * kvc_compact_pages without a caller-provided workspace, for callers that cannot allocate
 * device memory: engines whose allocator has given all free memory to the KV pool, or
 * foreign-function callers with no access to the host framework's allocator.  The pages
 * describe no such variant; it exists for those callers only.
 * Same arguments, checks and results as kvc_compact_pages, minus workspace/workspace_bytes:
 * the workspace is a fixed array inside the library (KVC_NOALLOC_MAX_ROWS + 1 int64 per
 * GPU, held from library load to process exit).  Calls for more than KVC_NOALLOC_MAX_ROWS
 * rows return KVC_ERR_UNSUPPORTED.  The first call on each device looks up the array's
 * device address (a synchronous runtime query).  All calls share the array, so calls
 * whose kernels can overlap on the GPU race and must be serialised by the caller.
 */
#define KVC_NOALLOC_MAX_ROWS 16384
kvc_status kvc_compact_pages_noalloc(const kvc_cache *cache, const int32_t *move_src, const int32_t *move_dst,
                                     const int32_t *num_moves, const int32_t *new_len, float *crf,
                                     int32_t *freed, int64_t freed_capacity, int64_t *num_freed,
                                     int32_t *d_status, kvc_stream_t stream);

/* bytes of device workspace kvc_append_tokens needs for `rows` rows */
size_t kvc_append_workspace_bytes(int32_t rows);

/*
 * Streaming a compacted cache forward ("KV-streams for Efficient Compaction in Agentic Reinforcement
 * Learning", abstract: the compacted cache is carried across rollouts instead of flushed and prefilled
 * again).  Appends `count` new tokens to every row: the K and V vectors of token i go to slot
 * row_len + i (i < count); where a row reaches a logical page it does not hold, it takes a page from the
 * top of the free-page stack (rows in order, each row's new pages in ascending logical order: row r's k-th
 * new page is free_pages[depth - total + offset_r + k], offset_r the pages all lower rows take, total the
 * pages of the call) and enters it in its block table; slot_pos = new_pos of the row's sequence,
 * slot_label = label, crf (when not NULL) = 0 for the new slots; row_len += count; *free_count -= total.
 * k_new, v_new: [rows][count][head_dim] in the cache dtype, 16-byte aligned; new_pos: [num_seqs][count]
 * int32; free_pages: the stack (e.g. kvc_compact_pages' freed list), *free_count (device int64, in/out) its
 * depth; workspace: kvc_append_workspace_bytes(rows) bytes of device memory.
 * Device faults: a stack too shallow for the call appends nothing and reports KVC_DEV_FREED_OVERFLOW
 * (row -1); a row that would exceed max_slots, or whose row_len is negative, is left alone and reported.
 */
kvc_status kvc_append_tokens(const kvc_cache *cache, const void *k_new, const void *v_new, const int32_t *new_pos,
                             int32_t count, uint8_t label, float *crf, int32_t *free_pages, int64_t *free_count,
                             void *workspace, size_t workspace_bytes, int32_t *d_status, kvc_stream_t stream);

/* bytes of the ratchet state buffer for num_seqs sequences */
size_t kvc_ratchet_state_bytes(int32_t num_seqs, const kvc_ratchet_params *params);

/* zero the state and set budget[seq] = state budget = params->init_budget */
kvc_status kvc_ratchet_init(void *state, int32_t *budget, int32_t num_seqs,
                            const kvc_ratchet_params *params, kvc_stream_t stream);

/*
 * Step 3 (monitor and ratchet), once per round: for each sequence and each of `steps`
 * decode steps, c_t = LSE(z_t) - mean of the top_k largest z_t (the average negative
 * log-probability of the top-k tokens).  Windows [stride*j, stride*j + window) over the
 * sequence's step stream (continuing across calls) are min-pooled as they complete;
 * pooled points whose window starts at or after the last expansion enter a least-squares
 * line y = a + b*j.  After the round, if at least min_points points are in the fit and
 * b < 0, budget <- min(floor(budget * grow_num / grow_den), cap), the fit restarts, and
 * the expansion step is recorded.  The budget never shrinks.
 * logits: [num_seqs][steps][vocab] fp32, vocab in [1, 2^24] (else KVC_ERR_UNSUPPORTED).
 * budget: [num_seqs] int32 (written).  confidence_out: [num_seqs][steps] fp32 c_t, or NULL.
 */
kvc_status kvc_confidence_ratchet(const float *logits, int32_t num_seqs, int32_t steps, int32_t vocab,
                                  void *state, int32_t *budget, float *confidence_out,
                                  const kvc_ratchet_params *params, int32_t *d_status,
                                  kvc_stream_t stream);

/*
 * Beacon queries ("BeaconKV Compresses KV Cache for Long-Reasoning Models with Beacon
 * Queries", Key ideas: revisit-related queries form a few similarity groups, a representative
 * of each group stands in for the query history, and these beacon queries join the recent
 * queries in the query set).  The page does not say how the groups are found; here each
 * group (sequence, layer, query head) keeps num_beacons beacons by online (mini-batch)
 * k-means, and every call folds in that group's new queries:
 *   1. beacons with count 0 are seeded, in index order, with the first new queries
 *      (the j-th empty beacon takes query j);
 *   2. every new query joins its nearest beacon among those with a count or a seed:
 *      squared Euclidean distance summed over d = 0..head_dim-1 in order, with the
 *      difference, the square and each partial sum rounded to fp32 separately (no fused
 *      multiply-add); the lower beacon index wins a tie;
 *   3. every beacon that drew new queries becomes the fp32 mean of all it has absorbed,
 *      in a fixed order: S = c * n, S += each of its new queries in query order,
 *      c = S / (n + drawn), n += drawn.  A beacon that drew nothing keeps its value (a seed
 *      that drew nothing keeps count 0 and is seeded afresh next call).
 * q:          new queries in the query-set layout [num_seqs][num_layers][max_q][num_q_heads]
 *             [head_dim], `dtype` KVC_BF16 or KVC_F32; sequence s brings num_q[s] of them
 *             (values above max_q are clamped, negative ones count as 0).
 * beacons:    [num_seqs][num_layers][num_q_heads][num_beacons][head_dim] fp32, in/out.
 * counts:     [num_seqs][num_layers][num_q_heads][num_beacons] int32, in/out; zero both
 *             arrays to start a group empty.
 * beacon_q:   NULL, or an output query set [num_seqs][num_layers][out_max_q][num_q_heads]
 *             [head_dim] in `dtype` whose rows 0..num_beacons-1 receive the beacons (rounded
 *             to nearest even for bf16), ready to lead the next round's query set; the
 *             other rows are not touched.
 * Limits: num_beacons in [1, 64], head_dim in [1, 256], max_q in [1, 65536], out_max_q >=
 * num_beacons; otherwise KVC_ERR_INVALID_ARGUMENT or KVC_ERR_UNSUPPORTED.  One CTA per group.
 */
kvc_status kvc_beacon_update(const void *q, const int32_t *num_q, int32_t num_seqs, int32_t num_layers,
                             int32_t num_q_heads, int32_t head_dim, int32_t max_q, kvc_dtype dtype,
                             float *beacons, int32_t *counts, int32_t num_beacons, void *beacon_q,
                             int32_t out_max_q, int32_t *d_status, kvc_stream_t stream);

/*
 * One decode step of paged attention with the step's score contribution folded in
 * ("ActKV Dissected", Component 3: the LSE is a byproduct of paged attention, so the
 * query's attention probabilities are its logits minus the LSE, with no gather of the
 * attention matrix and no recompute).  For every row (sequence, layer, KV head) and each
 * query head g of its GQA group, over the row's slots i < row_len with slot_pos <= q_pos:
 *     l[g, i] = q_g . k_i / sqrt(head_dim)
 *     lse[g]  = log sum_i exp(l[g, i])                  (-inf when no key is visible)
 *     out[g]  = sum_i exp(l[g, i] - lse[g]) v_i          (zeros when no key is visible)
 *     scores[row][i] (+)= sum_g exp(l[g, i] - lse[g])     (0 for a hidden slot)
 * q:       [num_seqs][num_layers][num_q_heads][head_dim] in the cache's dtype, one query
 *          per (sequence, layer, head); query head h belongs to KV head h / (num_q_heads /
 *          num_kv_heads).
 * q_pos:   [num_seqs] int32 position of the step's token (INT32_MAX sees every slot).
 * out:     [num_seqs][num_layers][num_q_heads][head_dim] fp32, written.
 * lse:     [num_seqs][num_layers][num_q_heads] fp32 natural log, written.
 * scores:  NULL (attention only) or [rows][max_pages_per_row * page_size] fp32, written
 *          (added to with KVC_SCORE_ACCUMULATE) for slots < row_len only.
 * flags:   0 or KVC_SCORE_ACCUMULATE.
 * Limits:  num_q_heads / num_kv_heads <= 8.  Each CTA of the row's cluster (at most 8 CTAs) keeps
 *          its slice's logits until the row's LSE is known, in one of two places (G' = the group
 *          size rounded up to a power of two):
 *          - tensor memory, when slot_pos and scores start on 16-byte boundaries, the page size
 *            has a divisor that is a multiple of 4, and either the cache is bf16 with 16-slot
 *            chunks and a 4-byte aligned q (any G'), or G' is 2 or 4 at head_dim 128 (2, 4 or 8
 *            at head_dim 64): the stages then also carry the chunk's positions and old scores,
 *            and every warp keeps two chunks in flight.  Rows up to 131,072 / 81,920 / 49,152
 *            slots at G' <= 2 / 4 / 8 with 16-slot chunks.  With bf16, 16-slot chunks and a
 *            4-byte aligned q, each chunk's q . k and probability-weighted V sums run on the
 *            tensor cores (fp32 accumulation; the probabilities enter as a bf16 pair that keeps
 *            16 bits of mantissa);
 *          - otherwise shared memory: (G' + 1) * 4 * ceil(max_slots / 8) bytes of logits and
 *            positions beside at least two K/V stages per warp, within 218 KiB; a stage holds a
 *            chunk of 16 slots of one page, shrinking to 8, 4, 2 or 1 slots (slower) when 16 do
 *            not fit.  For bf16 and head_dim 128, 16-slot chunks serve rows up to 92,416 / 61,568
 *            / 36,864 / 20,480 slots at G = 1 / 2 / 4 / 8.
 *          The longest rows accepted (the shared-memory bound, which the call checks whatever the
 *          pointers) are 215,040 / 143,360 / 82,736 / 42,320 slots at G = 1 / 2 / 4 / 8 for bf16
 *          and head_dim 128; longer ones return KVC_ERR_UNSUPPORTED.  d_status reports a bad page
 *          or a bad row length; the affected row's results are then undefined.
 * Every sum runs in a fixed order: results repeat bit for bit.  One cluster of up to 8 CTAs
 * per row, exchanging maxima, sums and partial outputs through distributed shared memory.
 */
kvc_status kvc_decode_attention(const kvc_cache *cache, const void *q, const int32_t *q_pos, int32_t num_q_heads,
                                float *out, float *lse, float *scores, uint32_t flags, int32_t *d_status,
                                kvc_stream_t stream);

/*
 * Step-aware ranking scores ("StepKV: Step-Aware KV Cache Compression for LLM Agents", abstract:
 * entries belong to the reasoning step that generated them, a step utility from the trajectory is
 * combined with token-level saliency, and the combined scores rank the prunable tokens under the
 * budget).  The page gives no formulas; computed here, for every row and slot i < row_len:
 *     step(i) = the last k with step_start[seq][k] <= slot_pos[i]
 *     U_k     = mean of scores[row][i] over the row's slots of step k
 *     out[row][i] = (1 - beta) * scores[row][i] + beta * U_step(i)
 * The result ranks entries through kvc_select_budget (pass it as the crf argument), in place of
 * or beside the LRFU values.
 * scores:     [rows][max_slots] fp32 token saliency (e.g. the step-1 scores).
 * step_start: [num_seqs][max_steps] int32 step start positions: step_start[s][0] = 0 and strictly
 *             ascending over the first num_steps[s] entries (steps begin where reasoning segments
 *             begin); a position maps to a step whatever slot the entry sits in, so the table
 *             stays valid across compactions.
 * num_steps:  [num_seqs] int32 in [1, max_steps].
 * max_steps:  in [1, 4096]; beta in [0, 1].
 * out:        [rows][max_slots] fp32, written for slots < row_len; may be the scores array itself.
 * Step sums are exact integer sums of the scores rounded to a per-row fixed point (max|s| * 2^-39),
 * so results repeat bit for bit.  d_status: KVC_DEV_BAD_STEPS, KVC_DEV_BAD_LENGTH, KVC_DEV_NONFINITE
 * for an infinite score (the row is left unwritten); a NaN score is not detected and leaves the
 * row's results undefined.  One CTA per row.
 */
kvc_status kvc_step_scores(const kvc_cache *cache, const float *scores, const int32_t *step_start,
                           const int32_t *num_steps, int32_t max_steps, float beta, float *out,
                           int32_t *d_status, kvc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
