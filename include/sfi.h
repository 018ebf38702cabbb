/*
 * sfi.h — C ABI of the Slow-Fast Inference (SFI) decode hot path on B200.
 *
 * Slow-Fast Inference ("Slow-Fast Inference: Training-Free Inference
 * Acceleration via Within-Sentence Support Stability", arXiv 2603.12038)
 * splits decoding into frequent cheap "fast" steps, which attend only to a
 * small sparse memory (sink tokens, Selector-chosen tokens packed into a
 * contiguous buffer, and a recent window read from the paged KV cache), and
 * occasional dense "slow" steps, whose attention distribution refreshes that
 * memory through the Selector.  Page sections cited below:
 *   [ES] gist.science/es "2. Metodología", "3. Optimización del Sistema"
 *   [FR] gist.science/fr "B. Le Sélecteur", "C. Optimisations Système"
 *   [NL] gist.science/nl "De Selector", "Systeemontwerp en Kernel-optimalisatie"
 *   [ZH] gist.science/zh "2.1", "2.2", "2.3"
 *
 * Conventions for every call:
 *  - Tensors are caller-owned device pointers; nothing is allocated on the
 *    decode path.  bf16 values are passed as raw 16-bit patterns (sfi_bf16).
 *  - Calls are asynchronous on the given CUDA stream (cudaStream_t passed as
 *    void*; NULL = legacy default stream) and return an sfi_status at once.
 *    Argument errors are reported before anything is enqueued.  Errors found
 *    on the device (an out-of-range page-table entry or index, a pipeline
 *    wait that timed out) skip the offending access and are latched into
 *    sfi_paged_kv.err (if non-NULL): low byte = sfi_status, next byte = the
 *    kernel site.  Read and clear it with sfi_poll_error().
 *  - Shapes: G = Hq / Hkv must be an integer in [1, 16]; D in {64, 128};
 *    page_size == 16.  The context length L (new token included) is passed
 *    by value and is the same for every sequence of the batch.
 *  - Device pointers handed to TMA (k_pool, v_pool, packed k/v) must be
 *    16-byte aligned.  Nothing here ever aborts or exits the process.
 *  - Consecutive calls on one stream overlap on the GPU: an attention call
 *    starts loading its query and cache rows, and a fast call appends its
 *    token, while earlier attention calls on the same stream finish.  So
 *    the query of an attention call must not be the output of an earlier
 *    attention call, and a fast call must not append to a cache row that an
 *    earlier call reads or appends, unless a kernel or copy of the caller's
 *    lies between the two calls on the stream (that orders them fully).  In
 *    a decode loop each layer has its own rows and other kernels produce the
 *    query.
 */
#ifndef SFI_H_
#define SFI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SFI_OK = 0,
  SFI_ERR_INVALID_ARG = 1,  /* NULL pointer, misaligned pointer, bad scalar */
  SFI_ERR_SHAPE = 2,        /* inconsistent or out-of-range sizes */
  SFI_ERR_UNSUPPORTED = 3,  /* valid but not built (e.g. D not in {64,128}) */
  SFI_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  SFI_ERR_DEVICE_CHECK = 5, /* a device-side bounds check fired */
  SFI_ERR_TIMEOUT = 6,      /* a device-side bounded wait expired */
  SFI_ERR_WORKSPACE = 7     /* workspace missing or too small */
} sfi_status;

typedef uint16_t sfi_bf16; /* raw bfloat16 bits */
typedef void* sfi_stream;  /* cudaStream_t */

/* Sizes of one attention layer.  B sequences, Hq query heads sharing Hkv KV
 * heads (G = Hq/Hkv query heads per KV group), head dim D.  The paged cache
 * has num_pages pages of page_size (=16) tokens per KV head; each sequence
 * owns max_pages entries of the page table. */
typedef struct {
  int32_t B, Hq, Hkv, D;
  int32_t page_size;
  int32_t max_pages;
  int32_t num_pages;
} sfi_shape;

/* Method constants (readings of the pages where they are silent):
 *  n_sink     sink tokens [0, n_sink), always attended        ([ES] §2)
 *  n_recent   recent window [L-n_recent, L), read from pages   ([ES] §2, [NL])
 *  k_fixed    >0: K per query head; else floor(budget_frac*L) ([ES] §4)
 *  lambda, lambda_clip   s = (1-l) f~ + l r, l = clamp(lambda, 0, lambda_clip)
 *                         ([NL] "De Selector", [ZH] §2.2, §4 ablations)
 *  alpha_soft, nms_window  soft-NMS strength and full window width (w = window/2)
 *  alpha_cross             cross-head exclusivity penalty      ([FR] §2.B)
 *  refresh_budget          M: a slow step at least every M steps ([ES] §2)
 *  evidence_window         W: the Selector's evidence averages the attention
 *                          distributions of the last W queries ([ES] §2, [ZH]
 *                          §2.2 "window"); 0 or 1: the slow step's query only.
 *                          W <= n_recent, W <= 32 and W * G <= 16. */
typedef struct {
  int32_t n_sink, n_recent, k_fixed;
  double budget_frac;   /* K = floor(budget_frac * L) in double precision */
  float lambda, lambda_clip, alpha_soft, alpha_cross;
  int32_t nms_window, refresh_budget;
  int32_t evidence_window;
} sfi_params;

/* The paged KV cache of one layer ([NL] "Systeemontwerp": the recent window is
 * read straight from it; [ZH] §2.3).
 *  k_pool, v_pool  bf16 [num_pages, Hkv, 16, D]; token j of sequence b, KV head
 *                  h is row j%16 of page page_table[b, j/16], head h.
 *  page_table      int32 [B, max_pages]
 *  key_norms       fp32  [B, Hkv, max_pages*16]: ||k_j||_2 of the stored bf16
 *                  key, the cache statistic the Selector's prior reads.
 *  err             int32 device word for latched device-side errors, or NULL. */
typedef struct {
  sfi_bf16* k_pool;
  sfi_bf16* v_pool;
  const int32_t* page_table;
  float* key_norms;
  int32_t* err;
} sfi_paged_kv;

/* Contiguous packed buffer of one layer ([ES] §3 item 2, [NL] Memory-Coalesced
 * Kernel, [ZH] §2.3): per (sequence, KV head) the sink rows, then the union of
 * the group's selected positions (ascending after sfi_compact; after
 * sfi_compact_incremental, rows that stayed selected keep their slots), then
 * zero rows up to a multiple of 16.  Readers treat the rows as a set.
 *  k, v      bf16  [B, Hkv, p_max, D]
 *  pos       int32 [B, Hkv, p_max]   cache position of each row
 *  headmask  uint32[B, Hkv, p_max]   bit h set: query head h of the group
 *                                     attends to this row (sinks: all bits)
 *  n_rows    int32 [B, Hkv]          rows in use (sinks included)
 *  p_max     row capacity, a multiple of 64 (see sfi_packed_rows). */
typedef struct {
  sfi_bf16* k;
  sfi_bf16* v;
  int32_t* pos;
  uint32_t* headmask;
  int32_t* n_rows;
  int32_t p_max;
} sfi_packed;

/* Optional outputs of the dense (slow-step) attention.  Any pointer may be
 * NULL.  Rows are [B, Hq, ld] with ld >= L (elements).
 *  lse        [B, Hq]  log sum_j exp(z_j), natural log, over [0, L)
 *  logits     z_j = q.k_j / sqrt(D) for j < L                ([ES] §2 "logits")
 *  probs      f_j = exp(z_j - lse) for j < L (may equal logits: in place;
 *             needs lse non-NULL)
 *  lse_cand   [B, Hq]  log sum_{j in [cand_lo, cand_hi)} exp(z_j); the
 *             Selector's evidence is f~_j = exp(z_j - lse_cand). */
typedef struct {
  float* lse;
  float* logits;
  float* probs;
  int64_t ld;
  float* lse_cand;
  int32_t cand_lo, cand_hi;
} sfi_dense_extras;

/* Text of a status code (static storage).  A utility of this library, no
 * step of the pages. */
const char* sfi_status_str(sfi_status s);

/* Library version string (static storage).  A utility, no step of the pages. */
const char* sfi_version(void);

/* Sizing calls (this and the next two): no step of the pages, they size the
 * caller's allocations for the steps below.
 * Bytes of scratch the per-op calls below need for contexts up to
 * L_max = max_pages * 16 tokens.  Pass at least that much as ws/ws_bytes
 * (16-byte aligned).  Ownership stays with the caller.  The scratch must be
 * zero-filled before its first use (the first 256 bytes hold a work counter
 * of the attention kernels, another part the incremental compaction's
 * previous-position bitmap); every
 * successful call leaves it ready for the next one (after an error, zero it
 * again).  Calls that share one ws must not run concurrently. */
sfi_status sfi_workspace_size(const sfi_shape* shape, const sfi_params* params, size_t* bytes);

/* Packed-buffer row capacity p_max needed for contexts up to max_pages*16:
 * n_sink + min(G*K_max, |C|_max), rounded up to a multiple of 64. */
sfi_status sfi_packed_rows(const sfi_shape* shape, const sfi_params* params, int32_t* p_max);

/* Selection size K for a slow step at context L: k_fixed or
 * floor(budget_frac * L), clamped to |C| = L - n_recent - n_sink.
 * Fails with SFI_ERR_SHAPE when |C| < 1. */
sfi_status sfi_budget(const sfi_params* params, int32_t L, int32_t* K);

/* Append one token per (sequence, KV head) at position L-1 and record its key
 * norm (fp64 sum of squares of the stored bf16 key, rounded once to fp32) when
 * kv->key_norms is non-NULL.  k_new, v_new: bf16 [B, Hkv, D], 16-byte aligned. */
sfi_status sfi_append_kv(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                         const sfi_bf16* k_new, const sfi_bf16* v_new, sfi_stream stream);

/* Recompute key_norms for positions [pos_lo, pos_hi) (e.g. after a prefill). */
sfi_status sfi_key_norms(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t pos_lo,
                         int32_t pos_hi, sfi_stream stream);

/* Slow-step dense decode attention over [0, L) ([ES] §2 Pasos Lentos; [FR] §2.A;
 * [ZH] §2.1), also the in-house full-KV baseline when extras == NULL.
 *  q    bf16 [B, Hq, D]; query head hq uses KV head hq / G.
 *  out  fp32 [B, Hq, D] = sum_j softmax(z)_j v_j.
 * Persistent split-K kernel: TMA page tiles -> shared memory, mma.sync for
 * the group's QK^T / PV tiles, online softmax, then a combine kernel. */
sfi_status sfi_dense_attn(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                          const sfi_bf16* q, float* out, const sfi_dense_extras* extras,
                          void* ws, size_t ws_bytes, sfi_stream stream);

/* sfi_append_kv and sfi_dense_attn in one launch: the work item of each
 * (b, kv head) that holds position L - 1 first writes k_new / v_new (bf16
 * [B, Hkv, D], 16-byte aligned) into that row of the pages and its key norm
 * into kv->key_norms (when non-NULL), then attends over [0, L) as
 * sfi_dense_attn does.  Results are those of the two calls in a row, bit for
 * bit; a page-table entry outside the pool is latched in kv->err
 * (SFI_ERR_DEVICE_CHECK) and that row is neither written nor attended.  The
 * pages fold the append into the decode step ([ES] §2; [ZH] §2.1) and do not
 * say how it is launched. */
sfi_status sfi_dense_attn_append(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                                 const sfi_bf16* k_new, const sfi_bf16* v_new, const sfi_bf16* q,
                                 float* out, const sfi_dense_extras* extras, void* ws, size_t ws_bytes,
                                 sfi_stream stream);

/* sfi_dense_attn without a workspace argument, for callers that cannot
 * allocate device memory where they call it: serving runtimes whose pool
 * hands the library only input and output tensors, and plugin or embedded
 * hosts without access to the CUDA allocator.  The paper has no counterpart
 * to this entry point.  Arguments, their checks and results are those of
 * sfi_dense_attn.  The scratch (a work
 * counter and the split-K partials) is a static 16 MiB device array that
 * every GPU loading the library holds until the process exits; a call whose
 * partials would not fit returns SFI_ERR_WORKSPACE and launches nothing.
 * Nothing is allocated.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress) and keeps it for the process, which
 * assumes the device's context is not reset meanwhile; make that first call
 * before any stream capture.  All calls share the one array and it keeps the last call's
 * contents (the counter is cleared at the start of every call): calls that
 * overlap on the GPU race, so order them (one stream, or events). */
sfi_status sfi_dense_attn_noalloc(const sfi_shape* shape, const sfi_paged_kv* kv, int32_t L,
                                  const sfi_bf16* q, float* out, const sfi_dense_extras* extras,
                                  sfi_stream stream);

/* f = exp(logits - lse) over j < L for every (b, hq) row: the attention
 * distribution itself, which [ZH] §2.2 names as the Selector's input (this
 * library's Selector reads the logits and lse_cand instead).  For callers
 * that want f; not on the decode path. */
sfi_status sfi_attn_probs(const sfi_shape* shape, int32_t L, const float* logits, int64_t ld,
                          const float* lse, float* probs, sfi_stream stream);

/* Fast-step sparse attention ([ES] §2 Pasos Rápidos; [NL] Methodologie):
 * query head h attends to the packed rows whose headmask has bit h (sinks +
 * its selection) and to the recent window [L - n_recent, L) read from pages.
 *  out fp32 [B, Hq, D]; lse fp32 [B, Hq] or NULL. */
sfi_status sfi_fast_attn(const sfi_shape* shape, const sfi_params* params,
                         const sfi_paged_kv* kv, int32_t L, const sfi_bf16* q,
                         const sfi_packed* packed, float* out, float* lse, void* ws,
                         size_t ws_bytes, sfi_stream stream);

/* sfi_append_kv and sfi_fast_attn in one launch (the step's token lies in the
 * recent window); append semantics, alignment and errors as for
 * sfi_dense_attn_append. */
sfi_status sfi_fast_attn_append(const sfi_shape* shape, const sfi_params* params,
                                const sfi_paged_kv* kv, int32_t L, const sfi_bf16* k_new,
                                const sfi_bf16* v_new, const sfi_bf16* q, const sfi_packed* packed,
                                float* out, float* lse, void* ws, size_t ws_bytes, sfi_stream stream);

/* Selector scores ([FR] "B. Le Sélecteur"; [NL] "De Selector"; [ZH] §2.2):
 * for the candidates C = [n_sink, L - n_recent) of a slow step at context L,
 * evidence f~ = exp(z - lse_cand), prior r from key norms and positions,
 * s = (1-l) f~ + l r, log-score, soft-NMS, cross-head exclusivity.
 *  logits    fp32 [B, Hq, ld] from sfi_dense_attn;  lse_cand fp32 [B, Hq]
 *  scores    fp32 [B, Hq, |C|] refined log-scores l''.
 * With W = params->evidence_window > 1 the evidence is the mean over W
 * queries of exp(z_i - lse_cand_i), and logits / lse_cand hold B x Hkv x W x G
 * rows: row ((b * Hkv + g) * W + i) * G + h is query i of head h of group g
 * (the layout sfi_dense_attn writes for a query tensor of Hkv * W * G heads
 * ordered that way). */
sfi_status sfi_select_scores(const sfi_shape* shape, const sfi_params* params,
                             const sfi_paged_kv* kv, int32_t L, const float* logits, int64_t ld,
                             const float* lse_cand, float* scores, void* ws, size_t ws_bytes,
                             sfi_stream stream);

/* Per-row top-K: the K largest of scores[r, 0:n] (finite values; ties ->
 * lower index), written ascending as idx[r, 0:K] = offset + column.  rows =
 * number of rows; scores row stride ld_s, idx row stride ld_i (elements);
 * n <= 262144, rows <= 65535.  The top-K keeps its state on chip and needs
 * no scratch: sfi_topk_workspace_size reports 0 and ws may be null (a
 * ws_bytes below the reported size is refused).  Exact radix select over
 * order-preserving 32-bit keys of the scores, one thread-block cluster of 1,
 * 2, 4 or 8 CTAs (of up to 1024 threads) per row, each CTA holding its
 * slice's keys on chip (32 per thread in registers, and 32 more in shared
 * memory when the rows would otherwise take more CTAs than the GPU has
 * SMs): the digit passes run over key - smallest key,
 * from the highest bit of (largest - smallest), at most 14 bits per pass; CTA
 * histograms meet in distributed shared memory, and the ties at the
 * threshold are taken in position order.  The pages name the step and give
 * no method: the Top-K of [FR] "B. Le Sélecteur" and [ZH] §2.2. */
sfi_status sfi_topk_workspace_size(int32_t rows, int32_t n, size_t* bytes);
sfi_status sfi_topk(int32_t rows, int32_t n, const float* scores, int64_t ld_s, int32_t K,
                    int32_t offset, int32_t* idx, int64_t ld_i, void* ws, size_t ws_bytes,
                    sfi_stream stream);

/* Full Selector = sfi_select_scores + sfi_topk.  sel_idx int32 [B, Hq, sel_ld]
 * receives K ascending absolute positions per query head; *K_out = K. */
sfi_status sfi_select(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv,
                      int32_t L, const float* logits, int64_t ld, const float* lse_cand,
                      int32_t* sel_idx, int32_t sel_ld, int32_t* K_out, void* ws,
                      size_t ws_bytes, sfi_stream stream);

/* Compaction ([ES] §3 item 2; [FR] §2.C "réorganisation"): build the packed
 * buffer of every (sequence, KV head) from the group's selections (K ascending
 * positions per query head, rows of sel_idx with stride sel_ld, all inside
 * the candidate range [n_sink, L - n_recent) of the slow step at context L)
 * by gathering K/V rows from the pages.  Bit-exact copies.  Rows beyond
 * p_max are dropped and reported as SFI_ERR_DEVICE_CHECK. */
sfi_status sfi_compact(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv,
                       int32_t L, const int32_t* sel_idx, int32_t sel_ld, int32_t K,
                       sfi_packed* packed, void* ws, size_t ws_bytes, sfi_stream stream);

/* Incremental compaction (the support of consecutive slow steps overlaps
 * strongly, "Slow-Fast Inference", within-sentence support stability): same
 * arguments and result set as sfi_compact, but `packed` must hold the previous
 * compaction of the same sequences and KV heads (by sfi_compact or this call,
 * same params, cache rows unchanged since), unless fresh != 0 or its n_rows is
 * 0.  Rows whose position stays selected keep their slot (head mask
 * rewritten); with U the new union and n_new = n_sink + |U|, the slots in
 * [n_sink, n_new) that are not kept receive, in slot order, the positions of
 * U not in the previous buffer (ascending) and then the kept rows at slots >=
 * n_new (in slot order), copied from the pages.  Rows [n_new, next multiple
 * of 16): zero, pos -1, mask 0.  A fresh buffer gets the layout of
 * sfi_compact.  packed->p_max must be at least the packed row capacity
 * (SFI_ERR_SHAPE otherwise).  ws as for sfi_select: zero-filled before its
 * first use, left so by every call. */
sfi_status sfi_compact_incremental(const sfi_shape* shape, const sfi_params* params, const sfi_paged_kv* kv,
                                   int32_t L, const int32_t* sel_idx, int32_t sel_ld, int32_t K,
                                   sfi_packed* packed, int32_t fresh, void* ws, size_t ws_bytes,
                                   sfi_stream stream);

/* Read the latched device error word of kv (synchronous), then clear it. */
sfi_status sfi_poll_error(const sfi_paged_kv* kv, int32_t* code);

/* Limit, in nanoseconds, of every device-side pipeline wait of the library's
 * kernels (process-wide; read at each launch; default 2e9).  A wait that
 * reaches it latches SFI_ERR_TIMEOUT with its site into the cache's error
 * word, stops waiting and lets its kernel return (copies in flight are
 * drained first, under a fixed 2 s limit), so the context stays usable.  The
 * limit must exceed the longest legitimate wait (milliseconds under heavy
 * load).  ns outside [1e5, 6e10]: SFI_ERR_INVALID_ARG.  Failure detection
 * has no counterpart in the pages. */
sfi_status sfi_set_wait_limit(int64_t ns);
sfi_status sfi_get_wait_limit(int64_t* ns);

/* Runs the library's bounded wait on a barrier that nothing completes, with
 * the given limit (ns in [1e3, 6e10]): the wait expires, SFI_ERR_TIMEOUT |
 * (11 << 8) is latched into kv->err (which must be non-NULL; no other field
 * is used) and the kernel returns.  For checking the expiry path on a healthy
 * GPU; asynchronous on stream.  No counterpart in the pages. */
sfi_status sfi_selftest_wait(const sfi_paged_kv* kv, int64_t limit_ns, sfi_stream stream);

/* ------------------------------------------------------------------------
 * Decode-step driver ([ES] §2 trigger, §3 item 1 asynchronous pipeline;
 * [ZH] §2.3 双 CUDA 流).  A context owns one side stream and per-layer events;
 * the caller owns every tensor and the context workspace.
 */
typedef struct sfi_ctx sfi_ctx;

/* L_max = shape->max_pages * 16 bounds every context length used with ctx. */
sfi_status sfi_ctx_create(const sfi_shape* shape, const sfi_params* params, int32_t n_layers,
                          int32_t overlap, sfi_ctx** out);
sfi_status sfi_ctx_destroy(sfi_ctx* ctx);
sfi_status sfi_ctx_workspace_size(const sfi_ctx* ctx, size_t* bytes);
sfi_status sfi_ctx_set_workspace(sfi_ctx* ctx, void* ws, size_t bytes);

/* Trigger ([ES] §2 Pasos Lentos; [ZH] §2.1 触发机制): step t is slow when
 * t == 0, or the previous step emitted a boundary token (boundary_prev != 0),
 * or t - last_slow >= refresh_budget.  Evaluated when layer == 0; the other
 * layers of the step reuse the decision.
 *
 * One layer of one decode step, enqueued on `stream` (the main stream):
 *  1. append k_new/v_new at position L-1 (key norm included);
 *  2. slow step: dense attention (+logits, lse_cand) -> out; then, on the
 *     side stream after an event, the Selector and compaction refresh this
 *     layer's packed buffer while the main stream moves on to layer+1;
 *     fast step: wait for this layer's pending refresh, then sparse attention
 *     over packed + recent -> out.
 *  q bf16 [B,Hq,D]; k_new, v_new bf16 [B,Hkv,D]; out fp32 [B,Hq,D].
 *  *was_slow (may be NULL) receives the step's decision (1 when any sequence
 *  is slow, after sfi_decode_step_rows on the same context). */
sfi_status sfi_decode_step(sfi_ctx* ctx, int32_t layer, int32_t step, int32_t boundary_prev,
                           int32_t L, const sfi_paged_kv* kv, sfi_packed* packed,
                           const sfi_bf16* q, const sfi_bf16* k_new, const sfi_bf16* v_new,
                           float* out, sfi_stream stream, int32_t* was_slow);

/* Compaction used by slow steps: incremental != 0 (the default) refreshes a
 * layer's packed buffer with sfi_compact_incremental's layout once that buffer
 * holds this context's previous refresh of the layer (the first slow step of
 * a layer, step 0, a new workspace or another packed buffer rebuild it
 * fully); 0: sfi_compact's full rebuild at every slow step. */
sfi_status sfi_ctx_set_compaction(sfi_ctx* ctx, int32_t incremental);

/* Per-sequence triggers ([ES] §2 Pasos Lentos: the boundary that makes a
 * step slow is a token of one sequence): sfi_decode_step with one trigger
 * per sequence.  boundary_prev: host int32 [B], sequence b emitted a boundary
 * token at the previous step (NULL: none).  At layer 0 every sequence b is
 * decided: slow when step == 0, boundary_prev[b] != 0, or step minus its last
 * slow step >= refresh_budget.  A step whose sequences are all slow (all
 * fast) runs as in sfi_decode_step; a mixed step runs, per layer, the dense
 * attention on the slow sequences (and, on the side stream, the Selector and
 * compaction of their packed buffers) and the fast attention on the others.
 * slow_rows: host int32 [B] receiving the decisions (may be NULL).  B <= 256
 * (SFI_ERR_UNSUPPORTED otherwise).  sfi_decode_step on the same context
 * applies its boundary flag to every sequence. */
sfi_status sfi_decode_step_rows(sfi_ctx* ctx, int32_t layer, int32_t step, const int32_t* boundary_prev,
                                int32_t L, const sfi_paged_kv* kv, sfi_packed* packed,
                                const sfi_bf16* q, const sfi_bf16* k_new, const sfi_bf16* v_new,
                                float* out, sfi_stream stream, int32_t* slow_rows);

/* Make `stream` wait for every outstanding side-stream refresh of ctx. */
sfi_status sfi_ctx_join(sfi_ctx* ctx, sfi_stream stream);

/* Per-kernel CUDA-event timing of the attention kernels launched by
 * sfi_decode_step (kind 0 = fast-attention main kernel, 1 = dense main
 * kernel).  A utility of this library, no step of the pages.
 * sfi_ctx_set_timing_layers(ctx, first, n): n = 0 off; n > 0 brackets the
 * attention launches of layers first, first + n, first + 2n, ... with an
 * event pair (an event between two launches keeps the second from starting
 * early, so sparse sampling leaves the other layers' launches overlapped).
 * sfi_ctx_set_timing(ctx, n) is the same with first = 0.  sfi_ctx_timing
 * synchronises on the recorded events and returns total milliseconds and
 * launch count since the last reset. */
sfi_status sfi_ctx_set_timing(sfi_ctx* ctx, int32_t layer_stride);
sfi_status sfi_ctx_set_timing_layers(sfi_ctx* ctx, int32_t first_layer, int32_t layer_stride);
sfi_status sfi_ctx_timing(sfi_ctx* ctx, int32_t kind, double* total_ms, int64_t* launches,
                          int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* SFI_H_ */
