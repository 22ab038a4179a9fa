/*
 * delta_attn.h — C ABI of the DELTA decode attention stack for NVIDIA B200 (sm_100a).
 *
 * DELTA ("DELTA: Dynamic Layer-Aware Token Attention for Efficient Long-Context
 * Reasoning", ai.info summary, section "Methodology in Plain English") splits a
 * model's layers into initial full-attention layers, a few delta-layers that run
 * full attention and rank the KV pages, and sparse layers that read only the pages
 * chosen by the most recent delta-layer.  The whole KV cache stays in memory, paged
 * 16 tokens to a page (same section).  This header
 * exposes one call per step of that decode path:
 *
 *   delta_kv_append    write the current token's k, v into the paged cache
 *                      (delta_kv_append_layers: every layer of a step in one launch)
 *   delta_full_attn    full decode attention (initial layers)
 *   delta_select_attn  full decode attention + per-page scores + page selection (delta-layers)
 *   delta_sparse_attn  decode attention over the selected pages only (sparse layers);
 *                      delta_sparse_attn_settled when the selection was final one kernel earlier
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument is DEVICE memory owned by the caller, except the
 *   descriptor structs themselves, which are read on the host during the call.
 *   The library allocates nothing and reads no environment variable.  Between
 *   calls it keeps only per-device caches filled on first use and never changed
 *   afterwards (SM count, kernel attributes it set, cluster occupancy, the driver's
 *   tensor-map encoder, the address of delta_full_attn_noalloc's scratch array),
 *   guarded by a mutex; a device reset (cudaDeviceReset) invalidates them, so
 *   reload the library after one.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   Every call only enqueues work: none synchronises the host, so every call can
 *   be captured in a CUDA graph.  Outputs are valid once the stream reaches them.
 * - Element type: DELTA_F32 (IEEE float) or DELTA_BF16 (bfloat16) for q, k, v, o;
 *   all arithmetic accumulates in fp32.
 * - Layouts (row-major, innermost last):
 *     q, o            [batch][num_q_heads][head_dim]
 *     k_new, v_new    [batch][num_kv_heads][head_dim]
 *     k_pool, v_pool  [num_phys_pages][num_kv_heads][page_size][head_dim]   (one pair per layer)
 *     page table      CSR: page_indptr[batch+1], page_indices[page_indptr[batch]] physical
 *                     page ids; logical page j of sequence b is page_indices[page_indptr[b]+j]
 *     kv_len          [batch] tokens of each sequence AFTER this step's append
 *                     (the current token is attended)
 *     sel_pages       [batch][sel_stride] ascending LOGICAL page ids, sel_cnt[batch] valid
 *     page_scores     [batch][max_pages_per_seq] fp32
 * - Grouped-query attention: query head h reads KV head h / (num_q_heads/num_kv_heads).
 * - Kernels are launched with programmatic dependent launch: a kernel may be scheduled while
 *   the previous kernel of the stream drains, and waits for it before reading q, the page
 *   holding each sequence's newest token, or a selection (delta_sparse_attn may load pages
 *   of the selection it finds before the wait, but uses them only if the selection read
 *   after the wait agrees).  The page table, kv_len and every other pool page are treated as
 *   inputs of the whole decode step and may be read before that wait, so a kernel that writes
 *   them must complete before the call (any kernel launched without programmatic dependent
 *   launch does).  delta_sparse_attn_settled reads everything but q before the wait.
 * - Host-detectable errors return a status and launch nothing.  A launch failure
 *   returns DELTA_ERR_CUDA.  Device-detected errors (a page id outside the pool, a
 *   kv_len beyond the sequence's pages, a selection entry outside the context, a
 *   wait that timed out) never trap: the offending access is skipped and a flag is
 *   raised in the workspace, which delta_read_device_error() reports.
 */
#ifndef DELTA_ATTN_H
#define DELTA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DELTA_OK = 0,
    DELTA_ERR_INVALID_ARG = 1,  /* null pointer, inconsistent sizes, misaligned buffer */
    DELTA_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels implement */
    DELTA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than delta_workspace_size() */
    DELTA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    DELTA_ERR_BOUNDS = 5        /* device-side check failed (reported by delta_read_device_error) */
} delta_status;

typedef enum { DELTA_F32 = 0, DELTA_BF16 = 1 } delta_dtype;

/* How per-token attention is aggregated over query heads for the page score. */
typedef enum {
    DELTA_HEAD_SUM = 0,  /* S_j = sum over query heads h and tokens t of page j of p[h][t] */
    DELTA_HEAD_MAX = 1   /* S_j = sum over tokens t of page j of max_h p[h][t] (the page's own rule: a
                            token's weight is its largest attention weight over the heads; ai.info summary,
                            "Methodology in Plain English"); needs delta_workspace_size_reduce(...,
                            DELTA_HEAD_MAX) */
} delta_head_reduce;

/* Shape of one attention layer.  Supported: head_dim 64 or 128, page_size 16,
 * num_q_heads a multiple of num_kv_heads with group size G = num_q_heads/num_kv_heads
 * in 1..8, num_kv_heads <= 64. */
typedef struct {
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t page_size;
    int32_t dtype;            /* delta_dtype */
    float   sm_scale;         /* logit scale; 0 selects 1/sqrt(head_dim) */
    int64_t num_phys_pages;   /* pages in each of k_pool / v_pool */
} delta_desc;

/* Paged-cache page table shared by every layer (device arrays, caller-owned). */
typedef struct {
    const int32_t* page_indptr;   /* [batch+1] */
    const int32_t* page_indices;  /* [page_indptr[batch]] physical page ids */
    const int32_t* kv_len;        /* [batch] tokens after the append, >= 0 */
    int32_t batch;                /* >= 0; 0 makes every call a no-op */
    int32_t max_pages_per_seq;    /* host-known upper bound on ceil(kv_len[b]/page_size) */
} delta_page_table;

/* Selection rule of a delta-layer (ai.info summary, "Main Findings" bullet 5 and
 * "Methodology in Plain English"): keep the pages overlapping the first sink_tokens
 * tokens and the last recency_tokens tokens, then add the budget_pages highest-scoring
 * remaining pages (equal scores: lower page index first). */
typedef struct {
    int32_t budget_pages;     /* k, >= 0 */
    int32_t sink_tokens;      /* >= 0 */
    int32_t recency_tokens;   /* >= 0 */
    int32_t reduce;           /* delta_head_reduce */
} delta_select_params;

/* Bytes of workspace any attention call below needs for this shape on the current
 * device.  The workspace is scratch owned by the caller; it must be 256-byte
 * aligned and zero-filled once (delta_workspace_init) before first use. */
size_t delta_workspace_size(const delta_desc* desc, int32_t batch, int32_t max_pages_per_seq);

/* Workspace for delta_select_attn with the given head reduction: DELTA_HEAD_MAX also keeps
 * every query head's per-token logits (batch * num_q_heads * max_pages_per_seq * 16 floats);
 * DELTA_HEAD_SUM needs exactly delta_workspace_size().  0 for an invalid reduce. */
size_t delta_workspace_size_reduce(const delta_desc* desc, int32_t batch, int32_t max_pages_per_seq,
                                   int32_t reduce);

/* Zero-fill a workspace (enqueued on `stream`). */
delta_status delta_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Minimum sel_stride: budget_pages + sink pages + recency pages (+1 for an unaligned end). */
int32_t delta_sel_capacity(const delta_select_params* sp, int32_t page_size);

/* Write token kv_len[b]-1 of every sequence: k_new[b][g] and v_new[b][g] go to slot
 * (kv_len[b]-1) % page_size of logical page (kv_len[b]-1) / page_size.  The page
 * must already be in the page table.  Sequences with kv_len 0 are skipped.  The
 * rest of the cache is never modified (DELTA evicts nothing from the cache; ai.info
 * summary, "Methodology in Plain English"). */
delta_status delta_kv_append(const delta_desc* desc, const delta_page_table* pt,
                             const void* k_new, const void* v_new,
                             void* k_pool, void* v_pool, void* stream);

/* The same append for every layer of a decode step in one launch: layer l copies k_new[l],
 * v_new[l] into k_pools[l], v_pools[l].  The four arguments are HOST arrays of num_layers
 * device pointers (num_layers <= 64; more gives DELTA_ERR_UNSUPPORTED); all layers share the
 * descriptor and the page table. */
delta_status delta_kv_append_layers(const delta_desc* desc, const delta_page_table* pt, int32_t num_layers,
                                    const void* const* k_new, const void* const* v_new,
                                    void* const* k_pools, void* const* v_pools, void* stream);

/* Full decode attention: o[b][h] = sum_t softmax_t(sm_scale * q[b][h].k_t) v_t over the
 * kv_len[b] cached tokens of KV head h/G (the initial layers of the stack; ai.info summary,
 * "Methodology in Plain English").  kv_len 0 gives o = 0. */
delta_status delta_full_attn(const delta_desc* desc, const delta_page_table* pt,
                             const void* q, const void* k_pool, const void* v_pool, void* o,
                             void* workspace, size_t ws_bytes, void* stream);

/* delta_full_attn without a workspace argument, for callers that cannot allocate device
 * memory themselves: code that runs inside a CUDA graph being captured or replayed, a
 * real-time loop that must never call cudaMalloc, or a host framework that owns every
 * allocation and exposes no allocator to plug-ins.  The paper has no counterpart; it is a
 * property of this library's interface.
 *
 * Same inputs, output and results as delta_full_attn.  Its scratch is a fixed 8 MiB array
 * inside the library (static device memory: every GPU that loads the library keeps it until
 * the process exits).  The call allocates and frees nothing.  Shapes whose
 * delta_workspace_size() exceeds 8 MiB return DELTA_ERR_UNSUPPORTED.
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *   with that device current; make that first call before any stream capture.
 * - All calls share the one array and it keeps the last call's contents: each call clears
 *   its counters first (cudaMemsetAsync on `stream`).  Calls whose kernels overlap on the
 *   GPU (other streams, other threads) race on the array and give wrong results; serialise
 *   them on one stream.
 * - Device-side check flags land in the shared array and are not reported; use
 *   delta_full_attn with a workspace to read them. */
delta_status delta_full_attn_noalloc(const delta_desc* desc, const delta_page_table* pt,
                                     const void* q, const void* k_pool, const void* v_pool, void* o,
                                     void* stream);

/* Delta-layer: the same output as delta_full_attn, plus the page selection of each
 * sequence.  Page score (HEAD_SUM): S[b][j] = sum over all query heads h and tokens
 * t of page j of the softmax probability p[h][t]; (HEAD_MAX) the sum over the page's
 * tokens of the maximum over heads of p[h][t].  Selection: sink pages, recency
 * pages and the budget_pages best remaining pages, written ascending to
 * sel_pages[b][0..sel_cnt[b]).  page_scores may be NULL; when given, S is written
 * for j < ceil(kv_len[b]/page_size).  sel_stride must be >= delta_sel_capacity().
 * max_pages_per_seq must be <= 32768 here.
 * HEAD_SUM runs as one kernel: the last CTA to finish among a sequence's CTAs scores
 * its pages and selects them (arrival counters in the workspace; no CTA waits).
 * HEAD_MAX adds a second kernel that scores every token.  The workspace's counters
 * return to zero at the end of every call; after a call that failed to launch or
 * was cut short, re-initialise the workspace (delta_workspace_init). */
delta_status delta_select_attn(const delta_desc* desc, const delta_page_table* pt,
                               const delta_select_params* sp,
                               const void* q, const void* k_pool, const void* v_pool, void* o,
                               int32_t* sel_cnt, int32_t* sel_pages, int32_t sel_stride,
                               float* page_scores,
                               void* workspace, size_t ws_bytes, void* stream);

/* Sparse layer: attention restricted to the tokens (< kv_len[b]) of the logical pages
 * sel_pages[b][0..sel_cnt[b]), softmax renormalised over them (the layers after a
 * delta-layer read only the pages it selected; ai.info summary, "Methodology in Plain
 * English").  Pages are mapped through the
 * page table, so one selection serves every layer's pools. */
delta_status delta_sparse_attn(const delta_desc* desc, const delta_page_table* pt,
                               const int32_t* sel_cnt, const int32_t* sel_pages, int32_t sel_stride,
                               const void* q, const void* k_pool, const void* v_pool, void* o,
                               void* workspace, size_t ws_bytes, void* stream);

/* delta_sparse_attn for a settled selection: the caller states that sel_cnt, sel_pages, the
 * pools and the page table were final before the kernel that precedes this call in `stream`
 * began (in a decode step: every sparse layer but the first after the delta-layer that wrote
 * the selection, since that first one directly follows the selection kernel).  The kernel
 * then reads the selection and loads its pages, the appended token's page included, before
 * waiting on the preceding kernel, instead of loading the selection again after the wait to
 * check a guess.  Same arguments, output, errors and device flags as delta_sparse_attn; a
 * call that breaks the statement may read a stale selection or page. */
delta_status delta_sparse_attn_settled(const delta_desc* desc, const delta_page_table* pt,
                                       const int32_t* sel_cnt, const int32_t* sel_pages, int32_t sel_stride,
                                       const void* q, const void* k_pool, const void* v_pool, void* o,
                                       void* workspace, size_t ws_bytes, void* stream);

/* Delta-layer calibration metric: shift_out[b] = 1 - cos(scores_a[b], scores_b[b]) over the
 * pages j < ceil(kv_len[b]/page_size) of two layers' page scores (the page_scores outputs of
 * delta_select_attn, [batch][max_pages_per_seq] fp32).  The calibration places delta-layers
 * where consecutive layers' attention differs most, the difference being one minus their
 * cosine similarity, averaged by the caller over steps and inputs (ai.info summary,
 * "Methodology in Plain English"); a layer's attention map is read as its page-score vector.
 * A zero vector gives a shift of 1. */
delta_status delta_layer_shift(const delta_page_table* pt, const float* scores_a, const float* scores_b,
                               float* shift_out, void* stream);

/* Delta-layer placement from calibration shifts (a HOST function: plain host arrays, no GPU
 * work).  shift[l] is the averaged shift between layers l-1 and l (delta_layer_shift, averaged by
 * the caller over steps and inputs).  The page fixes the first delta-layer (layer 2) and asks
 * for the rest at layers of large shift spread over the depth (ai.info summary, "Methodology in
 * Plain English" and "Main Findings", last bullet).  Rule: `first` opens the list; the layers
 * after it are taken by decreasing shift (equal shifts: lower layer first), each kept only when
 * at least min_gap layers from every layer already kept, until `count` are kept or none is left.
 * out_layers (host, room for max(count, 1) entries) receives them ascending, *out_count their
 * number.  DELTA_ERR_INVALID_ARG for null pointers, num_layers outside 1..4096, first outside
 * the layers, min_gap < 0 or a NaN shift. */
delta_status delta_choose_layers(const float* shift, int32_t num_layers, int32_t count, int32_t first,
                                 int32_t min_gap, int32_t* out_layers, int32_t* out_count);

/* Synchronise `stream`, read and clear the workspace's device error flags.
 * Returns DELTA_OK, DELTA_ERR_BOUNDS (a device-side check failed since the last
 * read) or DELTA_ERR_CUDA.  *flags_out (nullable) receives the raw flag bits:
 * 1 page id outside the pool, 2 kv_len beyond the sequence's pages, 4 selection
 * entry outside the context, 8 a wait timed out.  Not for the hot loop. */
delta_status delta_read_device_error(void* workspace, int32_t* flags_out, void* stream);

/* Static description of a status code. */
const char* delta_status_string(delta_status s);

#ifdef __cplusplus
}
#endif

#endif /* DELTA_ATTN_H */
