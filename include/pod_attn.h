/*
 * pod_attn.h -- C ABI of the fused hybrid-batch attention library (sm_100a).
 *
 * One hybrid batch = one prefill chunk (request 0: P new query tokens over C
 * earlier tokens, causal) plus B single-token decode requests, all reading one
 * paged KV cache.  The library runs both kinds of attention concurrently on the
 * same SMs from ONE persistent kernel whose CTAs read their SM id and take an
 * SM-local ticket that assigns them prefill or decode work, as in
 * "POD-Attention: Unlocking Full Prefill-Decode Overlap for Faster LLM
 * Inference" (explainer page, "How POD-Attention overlaps prefill and decode":
 * fuse into one kernel, self-assign roles per SM, 2 threadblocks per SM,
 * single-warp virtual decode blocks, capped KV splits, proportional allocation).
 * Split-KV partial results are combined by a log-sum-exp merge (the PAT
 * catalogue record merges its per-split results with online softmax), done by
 * the warp that finishes a row's last split.
 *
 * Math (per query head h, kv head h / (Hq/Hkv), natural-base softmax):
 *   prefill row i (absolute position C+i): O = softmax(scale q K[0..C+i]^T) V[0..C+i]
 *   decode request r:                      O = softmax(scale q K[0..L_r-1]^T) V[0..L_r-1]
 * bf16 operands, fp32 accumulation and softmax, bf16 outputs.
 *
 * Layouts (all row-major, element type bf16 unless stated):
 *   q_prefill   [P, Hq, d]                 o_prefill   [P, Hq, d]
 *   q_decode    [B, Hq, d]                 o_decode    [B, Hq, d]
 *   k_cache / v_cache  [num_blocks, Hkv, 16, d]  (one 16-token page of one kv
 *               head is contiguous); token j of a request lives in page
 *               block_table[row][j / 16], slot j % 16.
 *   block_table int32 [1 + B, block_table_stride]; row 0 = the prefill request
 *               (its kv length is C + P and its last P tokens are the chunk's own
 *               K/V, already written), row 1 + r = decode request r.
 *   kv_lens     int32 [1 + B] on the device: [0] = C + P, [1 + r] = L_r; the
 *               kernel checks them against the plan.
 *   Slots past a request's length in its last page may hold any FINITE value
 *   (the kernel zeroes masked V rows before use; K there is masked out).
 *
 * Ownership: the caller owns every device buffer (q, k/v cache, block table,
 * lengths, outputs, workspace, trace).  The library never allocates device
 * memory.  A plan is a host object owned by the library until
 * pod_attn_plan_destroy.
 *
 * Errors: every entry point returns an int status (POD_OK or a negative code);
 * nothing aborts or throws across the ABI.  Device-side problems found while
 * the kernel runs (block id out of range, a bounded wait that expired, lengths
 * that disagree with the plan) are recorded as a negative code in the int32
 * error word at byte offset pod_attn_plan_info.error_offset of the workspace
 * (the int32 after it holds the item or block involved); the offending access
 * is skipped (a load reads zeros), so no fault is raised.  Once a run has
 * completed in stream order, the word holds the first error of that run, or 0.
 */
#ifndef POD_ATTN_H_
#define POD_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  POD_OK = 0,
  POD_ERR_INVALID_ARG = -1,    /* bad sizes, lengths, null pointers, misalignment */
  POD_ERR_UNSUPPORTED = -2,    /* head_dim not 64/128, group > 8, page size not 16 */
  POD_ERR_WORKSPACE = -3,      /* workspace smaller than the plan needs */
  POD_ERR_CUDA = -4,           /* a CUDA runtime call failed (see pod_attn_last_cuda_error) */
  POD_ERR_BOUNDS = -5,         /* device: block id outside [0, num_blocks) */
  POD_ERR_TIMEOUT = -6,        /* device: a bounded wait expired; the kernel gave up */
  POD_ERR_PLAN_MISMATCH = -7   /* device: kv_lens disagree with the plan */
};

/* config.flags */
#define POD_FLAG_SEQUENTIAL 1u  /* ablation: prefill kernel, then decode kernel, then merge */
#define POD_FLAG_TRACE 2u       /* record the per-item schedule into `trace` */
#define POD_FLAG_MERGE_KERNEL 4u /* merge split-KV partials in a separate kernel after the attention
                                   kernel(s), instead of by the last split to finish inside them */
#define POD_FLAG_SELFTEST_TIMEOUT 8u /* diagnostic: CTA 0 first waits (1 ms limit) on a barrier that
                                       nothing arrives at, so the wait expires and POD_ERR_TIMEOUT is
                                       recorded in the error word; the attention itself still runs */
#define POD_FLAG_TWO_STREAMS 16u /* ablation: the prefill-only kernel on the caller's stream and the
                                    decode-only kernel on a library-owned stream forked from it and
                                    joined back with events (concurrent kernels, no co-location
                                    control); ignored with POD_FLAG_SEQUENTIAL */
#define POD_FLAG_SM_PARTITION 32u /* ablation of the per-SM tickets: in the fused kernel every CTA on
                                     one of the first ceil(prefill items / CTAs per SM) SM ids starts
                                     prefill-first and every other CTA decode-first (both still steal),
                                     so prefill and decode mostly run on separate SMs */
#define POD_FLAG_DECODE_FOUR_WARPS 64u /* ablation: only warps 0-3 of a decoding CTA run decode items
                                          (page rings 3 deep for d = 128, 4 for d = 64) and the plan's
                                          split cap counts 4 decode warps per CTA; by default all 6 warps
                                          decode (the MMA and TMA warps too; rings 2 / 3 deep) */
#define POD_FLAG_PREFILL_SPLIT_UNLIMITED 128u /* ablation: the prefill KV split fills every CTA slot even
                                                 when a short prefill (<= 1536 tokens) shares the batch
                                                 with decode work (the plan rule's co-located limit off,
                                                 which otherwise counts one prefill slot per SM) */

typedef struct pod_attn_config {
  int32_t num_q_heads;      /* Hq, 1..4096 */
  int32_t num_kv_heads;     /* Hkv; Hq % Hkv == 0 and Hq / Hkv <= 8 */
  int32_t head_dim;         /* d in {64, 128} */
  int32_t page_size;        /* tokens per KV page; must be 16 */
  int32_t num_sms;          /* 0 = query the current device */
  int32_t ctas_per_sm;      /* 0 = auto (2), 1 or 2 */
  int32_t ratio_prefill;    /* ticket ratio p:d; 0:0 = proportional rule */
  int32_t ratio_decode;
  int32_t max_waves;        /* split-KV cap in waves of decode warps; 0 = 2 */
  int32_t min_chunk_pages;  /* smallest split, in pages; 0 = 16 */
  int32_t max_prefill_splits; /* KV pieces per prefill item: 0 = the plan rule (at most 16), 1 = never
                                 split the prefill, 2..16 = the rule capped at this many */
  uint32_t flags;           /* POD_FLAG_* */
} pod_attn_config;

typedef struct pod_attn_plan pod_attn_plan_t;

typedef struct pod_attn_plan_info {
  int32_t num_prefill_items;  /* (128-row query tile, query head, key range) units */
  int32_t num_decode_items;   /* (request, kv head, key range) units */
  int32_t num_merge_items;    /* (request, kv head) rows with more than one split */
  int32_t num_partials;       /* split partial results held in the workspace */
  int32_t ctas_per_sm;
  int32_t ratio_prefill;
  int32_t ratio_decode;
  int32_t chunk_pages;        /* split size chosen by the plan, in pages */
  int32_t num_sms;
  int32_t grid;               /* CTAs of the persistent kernel */
  int64_t workspace_bytes;
  int64_t error_offset;       /* byte offset of the int32 device error word */
  int64_t prefill_flops;      /* 4 d Hq sum over every chunk row of the keys it sees */
  int64_t decode_flops;       /* 4 d Hq sum_r L_r */
  int64_t kv_bytes;           /* 4 d Hkv (sum_i (C_i + P_i) + sum_r L_r): K and V read once */
  int64_t qo_bytes;           /* 4 d Hq (sum_i P_i + B): Q read and O written once */
  int64_t table_bytes;        /* bytes pod_attn_upload copies host -> device */
  int32_t num_prefill_requests; /* NP: block-table / kv_lens rows 0..NP-1; decodes follow */
  int32_t num_prefill_rows;     /* sum_i P_i: rows of q_prefill / o_prefill */
  int32_t num_prefill_partials; /* KV pieces of split prefill items (partials in the workspace) */
  int32_t num_prefill_merge_items; /* prefill items cut into more than one KV piece */
  int64_t rescale_count_offset; /* byte offset of an int32 in the workspace that counts, with
                                   POD_FLAG_TRACE, the prefill softmax warps that rescaled O because
                                   a row max grew by more than 2^8 (diagnostic; 0 without the flag) */
} pod_attn_plan_info;

/* The plan rule.  The sources describe the knobs (explainer "How
 * POD-Attention overlaps prefill and decode": 2 threadblocks per SM, KV splits
 * capped at two full waves, CTAs in proportion to the prefill:decode mix;
 * FlashInfer PR "Limit kv split when prefill tokens <= 1536": the prefill's
 * split count leaves room for co-located decode CTAs) but give no formula;
 * this is the library's own rule, in integers throughout:
 *  - k = ctas_per_sm (0 -> 2); grid = num_sms * k.
 *  - Base prefill items: for request i (P_i rows over C_i earlier tokens), for
 *    query tile t = ceil(P_i/128)-1 .. 0, for head h: (q0 = 128 t, h,
 *    kv_end = C_i + min(128 (t+1), P_i), i) with n = ceil(kv_end/64) key tiles.
 *  - Decode split: cap = max_waves (0 -> 2) * num_sms * k * decode warps per
 *    CTA (6; 4 with POD_FLAG_DECODE_FOUR_WARPS); pages_r = ceil(L_r/16);
 *    c = max(min_chunk_pages (0 -> 16), ceil(Hkv sum pages_r / cap)), then
 *    c += 1 while c < max pages_r and Hkv sum ceil(pages_r / c) > cap.
 *    Request r is cut into S_r = ceil(pages_r / c) splits; split s covers
 *    pages [floor(s pages_r / S_r), floor((s+1) pages_r / S_r)).  Decode items
 *    are ordered by (pages descending, r, kv head, s); merge items follow
 *    (r, kv head) order; partial indices run over the split rows' items in
 *    (r, kv head, s) order.
 *  - Ticket ratio p:d: explicit ratios reduced by their gcd (a zero side gives
 *    1:0 or 0:1).  Otherwise 0:1 without prefill, 1:0 without decode, else
 *    cost_pre = prefill_flops, cost_dec = 248 * kv bytes of the decodes (248 =
 *    B200 tensor FLOP/s per HBM byte/s), tot = cost_pre + cost_dec,
 *    n_p = floor((2 k cost_pre + tot) / (2 tot)) clamped to [1, k-1] (k = 1:
 *    n_p = 1), and n_p = k when 2 cost_pre >= tot; p:d = n_p : k - n_p reduced.
 *  - Prefill KV split: limited = there are decodes and sum_i P_i <= 1536 and
 *    POD_FLAG_PREFILL_SPLIT_UNLIMITED is off; slots = num_sms if limited (one
 *    prefill slot per SM: the SM's other CTA stays for decode), else
 *    num_sms * k.  With n0 base items:
 *    if max_prefill_splits == 1 or n0 == 0 or n0 >= slots, nothing is split;
 *    else tau = max(8, ceil(sum n / slots)) and an item of n tiles gets
 *    S = min(smax, max(1, floor(n / tau))) pieces (smax = max_prefill_splits
 *    if >= 2, else 16), piece s covering key tiles [floor(s n/S),
 *    floor((s+1) n/S)).  Every piece spans at least 8 tiles.  Partial indices
 *    run over the pieces of split items in base-item order; prefill merge
 *    items (first partial, S) follow base-item order; all pieces are then
 *    stably ordered by key count, longest first.
 * The test oracle restates the same rule and the tests compare the two plans
 * bit for bit.
 *
 * Build the schedule for one hybrid batch on the host (no device work).
 * One prefill request: prefill_qo_len = P (0 = no prefill); prefill_kv_len = C + P
 * (ignored if P == 0); it owns block-table / kv_lens row 0 even when P == 0,
 * and decode request r owns row 1 + r.  decode_kv_lens = host array of B
 * lengths, each >= 1.  On success *plan_out owns a new plan and *workspace_bytes_out
 * (nullable) receives the device workspace size that pod_attn_upload /
 * pod_attn_run need.  Same as pod_attn_plan_batched with one prefill request.
 * Errors: POD_ERR_INVALID_ARG (also when a work count of pod_attn_plan_info
 * would not fit int64), POD_ERR_UNSUPPORTED, POD_ERR_CUDA (num_sms == 0 and no
 * device could be queried). */
int pod_attn_plan(const pod_attn_config* cfg, int32_t prefill_qo_len, int32_t prefill_kv_len,
                  int32_t num_decode, const int32_t* decode_kv_lens,
                  pod_attn_plan_t** plan_out, size_t* workspace_bytes_out);

/* Batched hybrid batch: num_prefill (0..4096) chunked-prefill requests and
 * num_decode decodes in one fused launch (the FlashInfer PR "Limit kv split when
 * prefill tokens <= 1536" times such a batched POD next to the one-prefill form).
 * Prefill request i (host arrays, length num_prefill): P_i = prefill_qo_lens[i]
 * query rows (0 allowed: the request has no work but keeps its row) over
 * prefill_kv_lens[i] = C_i + P_i keys, causal bottom-right; it owns block-table
 * / kv_lens row i, and its rows of q_prefill / o_prefill follow those of
 * requests 0..i-1.  Decode request r owns row num_prefill + r.  Rule, outputs
 * and errors as pod_attn_plan. */
int pod_attn_plan_batched(const pod_attn_config* cfg, int32_t num_prefill, const int32_t* prefill_qo_lens,
                          const int32_t* prefill_kv_lens, int32_t num_decode, const int32_t* decode_kv_lens,
                          pod_attn_plan_t** plan_out, size_t* workspace_bytes_out);

/* Copy the plan's summary into *info.  Errors: POD_ERR_INVALID_ARG (null). */
int pod_attn_plan_get_info(const pod_attn_plan_t* plan, pod_attn_plan_info* info);

/* Host copies of the work tables, for bit-exact checks; any pointer may be null.
 *   prefill_items int32 [num_prefill_items, 8]: q0 (row within its request), q_head,
 *                                               kv_end, prefill request, first and end key
 *                                               tile of the piece (64 keys per tile),
 *                                               partial (-1 = unsplit), prefill merge item
 *   decode_items  int32 [num_decode_items, 8]:  r, kv_head, k0, k1, partial (-1 = unsplit),
 *                                               merge item (-1 = unsplit), splits of the row, 0
 *   merge_items   int32 [num_merge_items, 4]:   r, kv_head, first_partial, num_splits */
int pod_attn_plan_tables(const pod_attn_plan_t* plan, int32_t* prefill_items,
                         int32_t* decode_items, int32_t* merge_items);

/* Copy the prefill merge table (host int32 [num_prefill_merge_items, 4]: first
 * partial, pieces, 0, 0) into `out` (nullable = skip).  Errors:
 * POD_ERR_INVALID_ARG (null plan). */
int pod_attn_plan_prefill_merges(const pod_attn_plan_t* plan, int32_t* out);

/* Copy the prefill request table (host int32 [num_prefill_requests, 4]: first
 * row of the request in q_prefill, P_i, C_i, 0) into `out` (nullable = skip).
 * Errors: POD_ERR_INVALID_ARG (null plan). */
int pod_attn_plan_prefill_requests(const pod_attn_plan_t* plan, int32_t* out);

/* Enqueue on `stream` (a cudaStream_t; NULL = legacy default stream) the
 * zeroing of the workspace's counters and the copy of the plan's work tables
 * into `workspace` (device, >= workspace_bytes, 256-byte aligned).  Call once
 * per plan and workspace before pod_attn_run (runs on the same plan and
 * workspace then need no further upload); the host tables may be destroyed
 * afterwards in stream order.
 * Errors: POD_ERR_INVALID_ARG, POD_ERR_WORKSPACE, POD_ERR_CUDA. */
int pod_attn_upload(const pod_attn_plan_t* plan, void* workspace, size_t workspace_bytes, void* stream);

/* Enqueue one hybrid-batch attention on `stream`: launch the persistent fused
 * kernel (or, with POD_FLAG_SEQUENTIAL in the plan's config, the prefill-only
 * then decode-only kernels; with POD_FLAG_TWO_STREAMS, the two on concurrent
 * streams, the call still completing in `stream` order).  The workspace's
 * ticket, queue and merge counters must be zero when a launch starts:
 * pod_attn_upload zeroes them, the fused kernel's last CTA returns them to zero
 * (so consecutive runs on one workspace need no clearing in between), and the
 * two-kernel and POD_FLAG_TRACE paths clear them with a memset first.  The
 * fused kernel is launched with programmatic stream serialization: its CTAs may
 * be scheduled while the previous kernel on `stream` finishes, and they wait for
 * that kernel to complete before reading or writing global memory.  Decode split-KV partials are merged by the warp that finishes a
 * row's last split (a completion counter, no waiting), or, with POD_FLAG_MERGE_KERNEL,
 * by the LSE merge kernel launched afterwards; the KV pieces of a split prefill item
 * are always merged by the CTA that finishes the item's last piece.  Asynchronous.
 * q/k/v/o pointers: device, 16-byte aligned; q_prefill / o_prefill hold the
 * prefill requests' rows one after another ([sum_i P_i, Hq, d]); unused sides
 * (no prefill rows, or B == 0) may be null.  block_table (device int32, row
 * stride block_table_stride) and kv_lens (device int32) have one row per
 * request: prefill requests first, then decodes.  num_blocks = pages in each
 * cache pool.  trace (nullable, used
 * with POD_FLAG_TRACE): int32 [num_prefill_items + num_decode_items, 4], zeroed
 * by the caller; entry = {smid, cta, home role (0 prefill, 1 decode), times run}.
 * Errors: POD_ERR_INVALID_ARG, POD_ERR_WORKSPACE, POD_ERR_CUDA (launch failed). */
int pod_attn_run(const pod_attn_plan_t* plan,
                 const void* q_prefill, const void* q_decode,
                 const void* k_cache, const void* v_cache, int64_t num_blocks,
                 const int32_t* block_table, int32_t block_table_stride,
                 const int32_t* kv_lens, float scale,
                 void* o_prefill, void* o_decode,
                 void* workspace, size_t workspace_bytes,
                 int32_t* trace, void* stream);

/* pod_attn_run with the decode requests reading an FP8 (e4m3) copy of the
 * paged cache: the KV bytes a decode streams are halved, which is the lever
 * the blog post "Prefill vs. Decode GPU Utilization Imbalance" names for the
 * bandwidth-bound decode ("Quantization and compression as a lever on both the
 * bandwidth and capacity problem").  The prefill requests keep reading the
 * bf16 pools (k_cache / v_cache, as in pod_attn_run; unused and nullable when
 * the plan has no prefill rows).
 *   k_cache_fp8 / v_cache_fp8  device uint8 [num_blocks_fp8, Hkv, 16, d], 16-byte
 *               aligned, e4m3 codes (1 sign, 4 exponent bits with bias 7, 3
 *               mantissa bits; no infinity, S.1111.111 is NaN); decode request r
 *               reads page block_table[NP + r][j / 16] of these pools.
 *   k_scale / v_scale  device float32 [Hkv]: the value of a stored code c of kv
 *               head h is k_scale[h] * e4m3(c) (v_scale for V).
 * Scores and P.V run on f16 tensor-core operands: e4m3 codes convert exactly,
 * and q_decode (bf16) is converted to f16, so its entries must lie within the
 * f16 range (|q| < 65504).  Slots past a request's length may hold any code,
 * NaN included (masked keys get no weight, masked V rows are zeroed).
 * Everything else (plan, workspace, flags, trace, errors) is as pod_attn_run. */
int pod_attn_run_fp8kv(const pod_attn_plan_t* plan,
                       const void* q_prefill, const void* q_decode,
                       const void* k_cache, const void* v_cache, int64_t num_blocks,
                       const void* k_cache_fp8, const void* v_cache_fp8, int64_t num_blocks_fp8,
                       const float* k_scale, const float* v_scale,
                       const int32_t* block_table, int32_t block_table_stride,
                       const int32_t* kv_lens, float scale,
                       void* o_prefill, void* o_decode,
                       void* workspace, size_t workspace_bytes,
                       int32_t* trace, void* stream);

/* Record `ev_start` / `ev_stop` (cudaEvent_t, nullable) on the stream around the
 * main attention kernel(s) of every later pod_attn_run with this plan (the
 * fused kernel; in sequential mode the prefill+decode kernels).  Lets a caller
 * time the dominant kernel without the counter reset and the merge. */
int pod_attn_plan_set_events(pod_attn_plan_t* plan, void* ev_start, void* ev_stop);

/* Helpers so callers without the CUDA headers can make timing events. */
int pod_attn_event_create(void** ev_out);
int pod_attn_event_destroy(void* ev);
int pod_attn_event_elapsed_ms(void* ev_start, void* ev_stop, float* ms_out);

/* Size of the fixed device workspace used by pod_attn_run_static (8 MiB). */
#define POD_STATIC_SCRATCH_BYTES (8u << 20)

/* pod_attn_run without a caller-provided workspace.  The paper has no
 * counterpart: this exists for callers that cannot allocate device memory,
 * such as a plugin inside an inference engine that keeps (almost) all HBM in
 * its own pools and offers no workspace hook, or a latency-critical caller
 * that cannot pay for cudaMalloc's implicit device synchronisation.
 * Instead of `workspace`, it uses a file-scope device array of
 * POD_STATIC_SCRATCH_BYTES that every GPU which loads the library holds until
 * the process exits; it allocates nothing.  Arguments, layouts and the async
 * behaviour are those of pod_attn_run (no trace).
 *  - Every call looks up the array's device address in the current context
 *    (cudaGetSymbolAddress), so the address stays right after cudaDeviceReset
 *    or in another context.  The first call in a context also loads the
 *    library's device code there; make that first call before any stream
 *    capture.
 *  - Every call re-copies the plan's tables (pod_attn_plan_info.table_bytes)
 *    into the array from the plan's pageable host copy, which can hold the
 *    host thread for the length of that copy, and zeroes the counters; the
 *    array keeps the last call's contents otherwise.
 *  - All calls on a device share the one array: calls that overlap on the GPU
 *    (other streams, other host threads) race and corrupt each other.
 *    Serialise them, e.g. on one stream.
 * Errors: POD_ERR_WORKSPACE if the plan needs more than
 * POD_STATIC_SCRATCH_BYTES (see pod_attn_plan_info.workspace_bytes); otherwise
 * those of pod_attn_upload and pod_attn_run. */
int pod_attn_run_static(const pod_attn_plan_t* plan,
                        const void* q_prefill, const void* q_decode,
                        const void* k_cache, const void* v_cache, int64_t num_blocks,
                        const int32_t* block_table, int32_t block_table_stride,
                        const int32_t* kv_lens, float scale,
                        void* o_prefill, void* o_decode, void* stream);

/* Release a plan (null is allowed). */
void pod_attn_plan_destroy(pod_attn_plan_t* plan);

/* Static text for a status code. */
const char* pod_attn_status_string(int status);

/* Last CUDA error code seen by the library in this thread (0 = none). */
int pod_attn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* POD_ATTN_H_ */
