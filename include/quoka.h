/*
 * quoka.h - C ABI of libquoka.so: query-oriented KV selection followed by sparse
 * attention for one chunk of a chunked LLM prefill, on one NVIDIA B200 (sm_100a).
 *
 * The problem statement follows the QUOKA page ("Qualcomm QuoKA ...", arXiv
 * 2602.08722): Figure 1(a) - every chunk of a chunked prefill first sub-selects the
 * KV cache, and the compacted cache is then fed to a dense attention kernel;
 * Figure 1(b) and the method summary - selection filters the chunk's queries by
 * cosine dissimilarity to their mean, scores keys by query-key cosine similarity,
 * and aggregates with max pooling over queries and mean pooling over the query
 * heads of a GQA group.  KV-head sharing (MQA / GQA) follows the "Multi-Query
 * Attention" page, technical insight section.  The QUILT page (shared-query
 * execution) motivates loading each selected K/V row once per chunk and reusing it
 * for every query of the group.
 *
 * Conventions for every call
 *   - All memory is owned by the caller.  The library allocates and frees nothing.
 *   - Device pointers must be 16-byte aligned; `workspace` must be 256-byte aligned.
 *   - Host arrays (kv_off, prefix_len, budget) are read before the call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Arguments are validated on the host before any launch: a failed
 *     check returns a non-OK status, launches nothing and leaves outputs untouched.
 *     quoka_last_error() then describes the failure (thread-local string).
 *   - Launch failures return QUOKA_ERR_CUDA.  Kernels never trap; a kernel that
 *     gives up a bounded wait records a nonzero code readable through
 *     quoka_device_error().
 *   - Tensor layouts (row-major, innermost dimension last):
 *       q_chunk  [batch, h_q, chunk, head_dim]               (dtype)
 *       k_cache  [h_kv, kv_off[batch], head_dim]             (dtype)
 *       v_cache  [h_kv, kv_off[batch], head_dim]             (dtype)
 *     Sequence b owns cache rows [kv_off[b], kv_off[b+1]).  Its prefix (the tokens
 *     of earlier chunks) is rows kv_off[b] .. kv_off[b]+prefix_len[b]-1, and the
 *     chunk's own K/V (already written by the caller) follow at
 *     kv_off[b]+prefix_len[b]+t for chunk position t.
 *   - Query head h uses KV head h / (h_q / h_kv).
 */
#ifndef QUOKA_H
#define QUOKA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QUOKA_OK = 0,
  QUOKA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or offset     */
  QUOKA_ERR_UNSUPPORTED = 2,   /* valid but unsupported: head_dim, batch, chunk    */
  QUOKA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required        */
  QUOKA_ERR_CUDA = 4           /* a CUDA runtime call or launch failed              */
} quoka_status;

typedef enum { QUOKA_F32 = 0, QUOKA_BF16 = 1 } quoka_dtype;

#define QUOKA_MAX_BATCH 64     /* sequences per call                                 */
#define QUOKA_MAX_CHUNK 8192   /* chunk tokens per sequence                          */
#define QUOKA_MAX_GROUP 64     /* query heads per KV head                            */

typedef struct {
  int batch;          /* sequences in this chunk step, 1..QUOKA_MAX_BATCH           */
  int h_q;            /* query heads                                                */
  int h_kv;           /* KV heads; h_q % h_kv == 0, h_q / h_kv <= QUOKA_MAX_GROUP   */
  int head_dim;       /* 64 or 128                                                  */
  int chunk;          /* C, chunk tokens per sequence, 1..QUOKA_MAX_CHUNK           */
  quoka_dtype dtype;  /* element type of q_chunk, k_cache, v_cache and out          */
} quoka_shape;

/*
 * Bytes of device scratch quoka_select() needs for prefixes up to `max_prefix` and
 * `nq` kept queries per head.  Returns 0 for an invalid shape.  The scratch holds
 * the gathered kept queries with their inverse norms and one fp32 pooled score per
 * prefix key and KV head (the full query-key score matrix is never stored).
 */
size_t quoka_select_workspace_size(const quoka_shape* shape, int max_prefix, int nq);

/*
 * Byte offset and row stride (in floats) of the pooled key scores inside the
 * workspace of quoka_select(): after a call, scores of sequence b, KV head g, key j
 * are at ((float*)(ws + offset))[(b * h_kv + g) * row_stride + j].  For tests and
 * diagnostics only.
 */
quoka_status quoka_workspace_pooled_view(const quoka_shape* shape, int max_prefix, int nq,
                                         size_t* offset, size_t* row_stride);

/*
 * quoka_select - QUOKA KV selection for one chunk step (QUOKA page: Figure 1(b) and
 * the method summary's three steps; Figure 2 for the direction of the query filter).
 *
 * Per sequence b and query head h, with C = shape->chunk, P = prefix_len[b]:
 *   1. m_h = mean over t < C of q_t / |q_t|                        (mean query)
 *   2. keep the Nk = min(nq, C) queries with the smallest cos(q_t, m_h), ties to the
 *      lower t                                                   (query subselection)
 * Per KV head g with heads H_g = {g*G .. g*G+G-1}, for every prefix key j < P:
 *   3. s_j = (1/G) * sum_{h in H_g} max_{i kept in h} cos(q_i, k_j)
 *                                  (cosine scoring; max then mean group pooling)
 *   4. keep the min(budget[b], P) keys with the largest s_j, ties to the lower j.
 * A zero-norm query or key has cosine 0.  The chunk's own keys are never candidates:
 * the attention call always adds them causally, so budget[b] counts prefix keys.
 * When every query is kept (nq >= chunk) and at most 16 query rows share a KV head (a
 * decode step, C = 1, or a short chunk), steps 1-2 are trivial and step 3 runs as a
 * stream over the keys (bf16: a 128 x 16 tensor-core MMA per 128-key tile; fp32: CUDA
 * cores); the result is the same.
 *
 *   q_chunk     device, [batch, h_q, chunk, head_dim]
 *   k_cache     device, [h_kv, kv_off[batch], head_dim]
 *   kv_off      host, batch + 1 nondecreasing row offsets, kv_off[0] >= 0,
 *               kv_off[b+1] - kv_off[b] >= prefix_len[b] + chunk
 *   prefix_len  host, batch entries, 0 <= P
 *   nq          kept queries per query head, >= 1 (values above chunk keep all)
 *   budget      host, batch entries, 0 <= budget[b] <= b_max
 *   b_max       row length of idx_out, >= 1
 *   idx_out     device int32 [batch, h_kv, b_max]: the kept prefix positions
 *               (relative to the sequence's first row) in ascending order, then -1
 *   kept_out    device int32 [batch, h_q, nq] or NULL: kept chunk positions in
 *               ascending order, then -1 when nq > chunk
 *   workspace   device scratch of quoka_select_workspace_size(shape, max_b P, nq)
 *               bytes; contents on entry are ignored
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE (ws_bytes too small), CUDA.
 */
quoka_status quoka_select(const quoka_shape* shape, const void* q_chunk, const void* k_cache,
                          const int64_t* kv_off, const int32_t* prefix_len, int nq,
                          const int32_t* budget, int b_max, int32_t* idx_out,
                          int32_t* kept_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * sparse_chunk_attn - dense attention of the chunk over the compacted cache
 * (QUOKA page, Figure 1(a): the compacted KV cache is fed to a dense attention
 * kernel; QUILT page: each shared K/V row is loaded once and reused by every query
 * that selected it - here the G query heads of a KV head share one selection).
 * For bf16 the call first writes that compacted cache (per sequence and KV head: the
 * selected rows, then the chunk's own rows) into `workspace`, then runs the dense
 * kernel over it; fp32 gathers rows directly and needs no workspace.  When at most 16
 * query rows share a KV head (G * chunk <= 16: a decode step, C = 1, or a short chunk;
 * QUOKA page, results summary: the method also serves the generation phase) both dtypes
 * instead gather the selected rows straight from the cache in a split-K kernel, whose
 * per-split partial results go in `workspace`, and merge the splits per KV head.
 *
 * Query t of head h (KV head g = h / G) of sequence b attends to
 *     keys  { idx[b, g, i] : i < n_b }  U  { P + u : 0 <= u <= t }
 * with n_b = min(budget[b], P) and P = prefix_len[b], computing
 *     out = softmax(q . k^T / sqrt(head_dim)) . v
 * with fp32 accumulation and fp32 softmax, stored in `dtype`.
 *
 *   q_chunk, k_cache, v_cache, kv_off, prefix_len   as for quoka_select
 *   budget      host, batch entries, 0 <= budget[b] <= b_max (as for quoka_select)
 *   idx         device int32 [batch, h_kv, b_max], e.g. quoka_select's idx_out;
 *               entries [0, n_b) must be distinct prefix positions in [0, P)
 *   out         device [batch, h_q, chunk, head_dim]; must not alias an input
 *   workspace   device scratch of sparse_chunk_attn_workspace_size(shape, b_max)
 *               bytes (may be NULL when that size is 0); contents on entry ignored
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.  An idx entry outside [0, P) is a
 * caller error; the kernels substitute a valid row for it and set a bit in the device
 * error word (quoka_device_error) instead of reading out of bounds.
 */
quoka_status sparse_chunk_attn(const quoka_shape* shape, const void* q_chunk,
                               const void* k_cache, const void* v_cache,
                               const int64_t* kv_off, const int32_t* prefix_len,
                               const int32_t* budget, const int32_t* idx, int b_max,
                               void* out, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device scratch sparse_chunk_attn() needs (0 if invalid; 0 for fp32 unless
 * G * chunk <= 16). */
size_t sparse_chunk_attn_workspace_size(const quoka_shape* shape, int b_max);

/*
 * sparse_perq_attn - attention where every query has its own selected keys, computed
 * with shared loading (QUILT page, summary: nearby queries are grouped, the key-value
 * entries they selected are loaded once and reused for all of them).
 *
 * Query t of head h of sequence b (KV head g = h / G) attends to exactly the positions
 * { sel[b, h, t, i] : i < S, sel[b, h, t, i] >= 0 } of its sequence's cache rows
 * (duplicates count once), out = softmax(q . k^T / sqrt(head_dim)) . v, fp32 softmax,
 * stored in `dtype`; a query whose set is empty gets zeros.  Causality is the caller's:
 * any position of the sequence may be listed.  Tiles of the G heads x (16 / G)
 * consecutive positions of a KV head load the union of their sets once.
 *
 *   q_chunk     device, [batch, h_q, chunk, head_dim]
 *   k_cache, v_cache  device, [h_kv, kv_off[batch], head_dim]
 *   kv_off      host, batch + 1 nondecreasing offsets, every sequence 1 .. 262144 rows
 *   sel         device int32 [batch, h_q, chunk, S]: positions relative to the sequence's
 *               first row, or -1; a position past the sequence sets the device error
 *               word and is ignored
 *   S           entries per query, 1 .. 2^20
 *   out         device, [batch, h_q, chunk, head_dim]; must not alias an input
 *   workspace   device scratch of sparse_perq_attn_workspace_size(shape, S) bytes
 * Limits: h_q / h_kv <= 16.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
quoka_status sparse_perq_attn(const quoka_shape* shape, const void* q_chunk,
                              const void* k_cache, const void* v_cache,
                              const int64_t* kv_off, const int32_t* sel, int S, void* out,
                              void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device scratch sparse_perq_attn() needs (0 if the arguments are invalid). */
size_t sparse_perq_attn_workspace_size(const quoka_shape* shape, int S);

/*
 * sparse_perq_attn_tc - sparse_perq_attn on tensor cores, for sets that the rows of a
 * tile largely share (QUILT page, summary: the shared entries are loaded once, and the
 * sharing is organised to fit the accelerator's tiles).
 *
 * Same result and arguments as sparse_perq_attn (sel rows in any order, duplicates count
 * once, -1 ignored, empty sets give zeros), computed per pair tile of 256 query rows: the
 * G heads of a KV head at 2 x (128 / G) consecutive positions.  The tile's sets are merged
 * into one union of keys (ascending), whose K/V rows are gathered once; dense 256-row
 * tcgen05 MMAs compute the logits of every row against every union key, and a per-row
 * membership mask keeps only the row's own keys in its softmax.  The work per tile grows
 * with its union, so this pays when the union is a small multiple of S.
 *   max_union   bound on any tile's union (1 .. about 40000, fixed by the masks' shared
 *               memory); sizes the workspace.  A tile whose union is larger sets bit 3 of
 *               the device error word and keeps only its first max_union keys (that
 *               tile's result is then wrong).
 *   workspace   sparse_perq_attn_tc_workspace_size(shape, S, max_union) bytes
 * Limits: bf16, head_dim 128, sequences of 1 .. 262144 rows.  Errors: INVALID_ARG,
 * UNSUPPORTED, WORKSPACE, CUDA.
 */
quoka_status sparse_perq_attn_tc(const quoka_shape* shape, const void* q_chunk,
                                 const void* k_cache, const void* v_cache,
                                 const int64_t* kv_off, const int32_t* sel, int S, int max_union,
                                 void* out, void* workspace, size_t ws_bytes, void* stream);
size_t sparse_perq_attn_tc_workspace_size(const quoka_shape* shape, int S, int max_union);

/*
 * quoka_step - one step of a chunked prefill or of decode, the way a serving loop runs
 * it: the chunk's new K/V rows go into the cache inside the call, then quoka_select and
 * sparse_chunk_attn run as described above (QUOKA page, Figure 1(a): each chunk sub-
 * selects the cache written before it, then attends over the compacted cache).
 *
 * For every sequence b the chunk's K/V rows are written to cache rows
 * kv_off[b] + prefix_len[b] + t (for bf16 inside the compaction pass that the attention
 * makes anyway).  The selection reads only rows below prefix_len[b], so the result
 * equals appending the rows by hand and calling quoka_select and sparse_chunk_attn.
 * The selection is skipped when no sequence keeps a prefix key.
 *
 *   q_chunk, kv_off, prefix_len, nq, budget, b_max   as for quoka_select
 *   k_new, v_new  device, [batch, h_kv, chunk, head_dim]: the chunk's keys and values
 *   k_cache, v_cache  device, [h_kv, kv_off[batch], head_dim]; rows kv_off[b] +
 *               prefix_len[b] .. + chunk - 1 are written, other rows untouched
 *   idx         device int32 [batch, h_kv, b_max]: the selection (written when one runs)
 *   out         device [batch, h_q, chunk, head_dim]; must not alias an input
 *   workspace   device scratch of quoka_step_workspace_size(shape, max_b prefix_len[b],
 *               nq, b_max) bytes; contents on entry ignored
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA; a failed check launches nothing.
 */
quoka_status quoka_step(const quoka_shape* shape, const void* q_chunk, const void* k_new,
                        const void* v_new, void* k_cache, void* v_cache,
                        const int64_t* kv_off, const int32_t* prefix_len, int nq,
                        const int32_t* budget, int b_max, int32_t* idx, void* out,
                        void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device scratch quoka_step() needs (0 if the arguments are invalid). */
size_t quoka_step_workspace_size(const quoka_shape* shape, int max_prefix, int nq, int b_max);

/*
 * quoka_prefill - a whole prompt through chunked prefill, chunk after chunk, with the
 * KV cache append inside the call (QUOKA page, Figure 1(a): the prompt is cut into
 * chunks of C tokens; each chunk first sub-selects the cache built by the chunks before
 * it and then runs dense attention over the compacted cache; the page's results
 * summary reports the time to first token this loop saves on NVIDIA GPUs).
 *
 * Every sequence of the batch holds a prompt of n_chunks * C tokens.  For chunk
 * c = 0 .. n_chunks-1, with P = c * C:
 *   1. this chunk's K/V rows are written to cache rows kv_off[b] + P + t (for bf16
 *      inside the compaction pass that the attention makes anyway, so the rows are
 *      read from k_new / v_new once);
 *   2. if c > 0 and budgets[c] > 0: quoka_select over the P prefix rows;
 *   3. sparse_chunk_attn of the chunk's queries, with budget[b] = budgets[c].
 * Chunk c's output equals quoka_select + sparse_chunk_attn called by hand with
 * prefix_len = c * C after the caller appended chunk c's rows.
 *
 *   n_chunks    chunks in the prompt, >= 1
 *   q           device, [n_chunks, batch, h_q, chunk, head_dim]
 *   k_new       device, [n_chunks, batch, h_kv, chunk, head_dim]: the prompt's keys
 *   v_new       device, [n_chunks, batch, h_kv, chunk, head_dim]: the prompt's values
 *   k_cache     device, [h_kv, kv_off[batch], head_dim]; written: rows kv_off[b] ..
 *               kv_off[b] + n_chunks*C - 1 of every KV head; other rows are untouched
 *   v_cache     device, as k_cache
 *   kv_off      host, batch + 1 nondecreasing row offsets, kv_off[0] >= 0,
 *               kv_off[b+1] - kv_off[b] >= n_chunks * chunk
 *   nq          kept queries per query head, >= 1
 *   budgets     host, n_chunks entries, 0 <= budgets[c] <= b_max: prefix keys each
 *               chunk keeps (chunk 0 has no prefix and ignores its entry)
 *   b_max       row length of idx, >= 1
 *   idx         device int32 [batch, h_kv, b_max]: scratch for the selections; holds
 *               the last chunk's selection after the call (if it ran one)
 *   out         device, [n_chunks, batch, h_q, chunk, head_dim]; must not alias an input
 *   workspace   device scratch of quoka_prefill_workspace_size(shape, n_chunks, nq,
 *               b_max) bytes; contents on entry ignored
 * All arguments are checked before the first launch; a failed check launches nothing.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
quoka_status quoka_prefill(const quoka_shape* shape, int n_chunks, const void* q,
                           const void* k_new, const void* v_new, void* k_cache,
                           void* v_cache, const int64_t* kv_off, int nq,
                           const int32_t* budgets, int b_max, int32_t* idx, void* out,
                           void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device scratch quoka_prefill() needs (0 if the arguments are invalid). */
size_t quoka_prefill_workspace_size(const quoka_shape* shape, int n_chunks, int nq, int b_max);

/*
 * Selected-value cache with miss-only fetch (SQD page, the paragraph on sparse
 * attention: the top-k choice still scans the whole cache where the cache lives, and
 * attention over the chosen positions runs elsewhere; the chosen values are kept there
 * and only the misses are sent, ahead of time).
 *
 * The cache keeps, per (sequence, KV head), the K/V rows of the current selection in a
 * block laid out as the attention kernels read it: `kc_rows` = (b_max + chunk) rounded
 * up to a multiple of 128 rows; slots 0 .. n-1 (n = min(budget[b], prefix_len[b])) hold
 * the selected prefix rows in slot order, slots n .. n+chunk-1 the chunk's own rows
 * (cache rows prefix_len[b] + t), then zero rows up to the next multiple of 128.
 *   sel_cache  device, caller-owned, quoka_selcache_bytes() bytes, 256-byte aligned:
 *              all K blocks [batch][h_kv][kc_rows][head_dim], then all V blocks, in
 *              the shape's dtype.
 *   slot_rows  device int32 [batch][h_kv][b_max], caller-owned: the row (relative to
 *              the sequence's kv_off) that each slot holds, -1 for none.  Fill it with
 *              -1 before the first update; afterwards only the updates write it.
 * One cache serves one shape (batch, h_kv, head_dim, chunk, dtype) and one b_max.
 *
 * quoka_selcache_update - bring the cache to a new selection `idx` (as quoka_select
 * writes it: [batch][h_kv][b_max], n ascending rows < prefix_len[b], then -1).  A row
 * the cache already holds in a slot below n stays in that slot (a hit: no copy); the
 * rows it does not hold (the misses) are copied from k_cache / v_cache into the slots
 * that fell free, the k-th miss in ascending row order into the k-th free slot in
 * ascending slot order; slots at or past n are emptied; the chunk rows and the zero
 * rows are rewritten.  `misses` (device int32 [batch][h_kv], or NULL) receives the
 * number of rows fetched per (sequence, KV head).  Arguments as for quoka_select; the
 * workspace (quoka_selcache_workspace_size() bytes) is scratch.  The longest prefix and
 * b_max must fit one shared-memory bitmap each (prefix + b_max up to about 900K rows);
 * longer calls return QUOKA_ERR_UNSUPPORTED.  Asynchronous on `stream`; an index outside
 * [0, prefix_len) sets the device error word (quoka_device_error) and is skipped.
 *
 * sparse_chunk_attn_selcache - the attention of sparse_chunk_attn, reading the selected
 * and the chunk's K/V rows from the cache instead of gathering them from the KV cache:
 * query t of head h attends to the n slots of KV head h / G and to chunk slots n .. n+t.
 * The result is the attention over the set of rows the slots hold; it is bit-identical
 * to sparse_chunk_attn over the same selection when the slots hold the rows in ascending
 * order (after an update from an empty cache, or one with no miss from such a state), and
 * equal up to the order of floating-point summation otherwise.  The workspace is the
 * same size as the update's.
 */
size_t quoka_selcache_bytes(const quoka_shape* shape, int b_max);
size_t quoka_selcache_workspace_size(const quoka_shape* shape, int b_max);
quoka_status quoka_selcache_update(const quoka_shape* shape, const void* k_cache, const void* v_cache,
                                   const int64_t* kv_off, const int32_t* prefix_len,
                                   const int32_t* budget, const int32_t* idx, int b_max,
                                   void* sel_cache, int32_t* slot_rows, int32_t* misses,
                                   void* workspace, size_t ws_bytes, void* stream);
quoka_status sparse_chunk_attn_selcache(const quoka_shape* shape, const void* q_chunk,
                                        const int32_t* prefix_len, const int32_t* budget,
                                        const void* sel_cache, int b_max, void* out,
                                        void* workspace, size_t ws_bytes, void* stream);

/*
 * quoka_select_noalloc - quoka_select without a caller-provided workspace.
 *
 * The paper has no counterpart to this call; it exists for callers that cannot
 * allocate device memory at the point where they run the selection: for example a
 * plugin inside a serving engine that reserved nearly all HBM for its KV cache at
 * start-up and hands plugins no allocator, or a latency-critical path where the
 * device synchronisation implied by cudaMalloc/cudaFree is not acceptable.
 *
 * Same arguments, semantics and errors as quoka_select, minus workspace/ws_bytes.
 * The scratch lives in one fixed device array of QUOKA_NOALLOC_SCRATCH_BYTES inside
 * the library, reserved on every GPU that loads the library until the process
 * exits.  A call whose quoka_select_workspace_size() would exceed that size returns
 * QUOKA_ERR_WORKSPACE and launches nothing.  The first call on a device looks up the
 * array's device address (once per device and context, with that device current);
 * make that first call before any stream capture.  After cudaDeviceReset the next
 * call sees a new context and looks the address up again.  All calls share the one array and the
 * kernels overwrite every scratch byte they read, so nothing needs clearing between
 * calls - but two calls whose kernels overlap on the GPU (different streams without
 * ordering between them) race on the array.  The library allocates nothing here.
 */
#define QUOKA_NOALLOC_SCRATCH_BYTES (32u << 20)
quoka_status quoka_select_noalloc(const quoka_shape* shape, const void* q_chunk,
                                  const void* k_cache, const int64_t* kv_off,
                                  const int32_t* prefix_len, int nq, const int32_t* budget,
                                  int b_max, int32_t* idx_out, int32_t* kept_out, void* stream);

/*
 * quoka_profile_events - per-kernel timing, for diagnostics and benchmarks.
 *
 * The paper has no counterpart to this call.  `events` is an array of `n_events`
 * caller-created CUDA events (cudaEvent_t handles created with timing enabled and
 * already valid on the device of the calls), or NULL to stop.  While an array is set
 * on the calling thread, every kernel the library launches from that thread is
 * followed by a cudaEventRecord of the next unused event on the launch's stream, until
 * all n_events are used; a caller that records its own event on the stream before a
 * call gets each kernel's time as the gap between consecutive events.  The caller owns
 * the events (the library only records them) and must keep the array alive while it
 * is set.  Do not set an array while capturing a stream into a graph.  Setting an
 * array, or NULL, resets the count.  Returns QUOKA_ERR_INVALID_ARG for n_events < 1
 * or a NULL handle.
 */
quoka_status quoka_profile_events(void* const* events, int n_events);

/*
 * How many events the launches recorded since quoka_profile_events on this thread;
 * names[i] (for i < max_names; names may be NULL) receives the name of the kernel whose
 * launch recorded event i (static strings owned by the library).
 */
int quoka_profile_marks(const char** names, int max_names);

/* Thread-local description of the last non-OK status returned on this thread. */
const char* quoka_last_error(void);

/*
 * Reads and clears the device error word (0 = none): bit 0 a bounded wait gave up, bit 2
 * an index outside its range, bit 3 a per-query tile's union over max_union.
 * Synchronises `stream`.  Returns QUOKA_ERR_CUDA if the read itself fails.
 */
quoka_status quoka_device_error(uint32_t* code, void* stream);

/* Library ABI version (major * 100 + minor). */
int quoka_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QUOKA_H */
