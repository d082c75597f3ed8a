/*
 * pa.h -- C ABI of the B200 (sm_100a) paged-KV grouped-query attention engine.
 *
 * The engine computes, for a batch of variable-length requests whose keys and
 * values live in a shared page pool,
 *
 *     O = softmax(scale * Q K^T + causal mask) V,   LSE = ln sum exp(scale * Q K^T)
 *
 * in one launch sequence that covers decode (one query token per request),
 * causal paged prefill and mixed batches of both.
 *
 * Sources for the contract:
 *  - "integrate PrimTS FMHA kernels" (TensorRT-LLM PR #17399), section
 *    "Unified page-table metadata": an int32 row-strided page table [B, C]
 *    plus live int32 seq_lens[B]; logical page p of request b is
 *    page_table[b][p]; columns past ceil(seq_lens[b] / page_size) are never
 *    read.  Section "Planning, preprocessing, and workspace ownership": one
 *    plan per active batch size, geometry and capacity fixed in the plan,
 *    request metadata bound at run time; only a split counter is reset per
 *    run.  Section "Integration and supported scope": page sizes
 *    16/32/64/128, head dims 64/128/256, GQA ratio up to 32, fail closed on
 *    anything else.
 *  - "Unified Triton kernel that doesn't distinguish between prefill +
 *    decode" (vLLM PR #16828): varlen packed queries addressed by cu_q_lens
 *    (like flash_attn_varlen_func), GQA query heads packed along the query
 *    dimension, causal mask applied by select to -inf.
 *  - "[Perf][FA4] Warm up dense (paged) FA4 attention kernels" (vLLM PR
 *    #48156), review thread: split-KV decode (num_splits > 1, 0 = automatic)
 *    and CUDA-graph (FULL) decode, hence pa_run must be capturable.
 *
 * Conventions of every entry point:
 *  - Pointers named as device pointers must point to memory of the current
 *    CUDA device; they are owned by the caller and only read or written during
 *    the stream work that pa_run enqueues.
 *  - Integer return codes: PA_OK (0) on success, otherwise a PA_ERR_* value;
 *    pa_last_error() then describes the failure (thread-local string, valid
 *    until the next call on the same thread).
 *  - A plan is not safe for concurrent use from several streams or threads:
 *    its workspace is shared by all runs.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *pa_stream_t;

typedef struct pa_plan pa_plan; /* opaque; owns the device workspace */

enum {
    PA_OK = 0,
    PA_ERR_INVALID = 1,     /* NULL or misaligned pointer, bad argument value */
    PA_ERR_UNSUPPORTED = 2, /* geometry outside the supported envelope */
    PA_ERR_CUDA = 3         /* a CUDA runtime call or launch failed */
};

/* Bits of the sticky device status word (pa_get_status).  The kernels never
 * trap and never wait on the host; they record bad request data here and
 * carry on with a defined fallback for the affected rows. */
enum {
    PA_STATUS_BAD_PAGE = 1u << 0,     /* a live page id < 0 or >= num_pages: that
                                         page reads as zeros, outputs of the request
                                         are unspecified */
    PA_STATUS_Q_GT_KV = 1u << 1,      /* q_b > seq_lens[b]: rows that see no key get
                                         O = 0, LSE = -inf */
    PA_STATUS_KV_GT_CAPACITY = 1u << 2, /* seq_lens[b] > capacity * page_size or < 0:
                                         clamped into [0, capacity * page_size] */
    PA_STATUS_BAD_CU_Q = 1u << 3,     /* cu_q_lens decreasing or cu_q_lens[0] != 0:
                                         the request is treated as having no tokens */
    PA_STATUS_TIMEOUT = 1u << 4       /* an internal pipeline wait ran out (never
                                         expected); the launch returned early */
};

/*
 * pa_create_plan -- validate a geometry and allocate the plan's workspace.
 *
 *   batch       B, number of requests each pa_run covers (> 0)
 *   heads_q     Hq, query heads (> 0, multiple of heads_kv)
 *   heads_kv    Hkv, KV heads (> 0); GQA ratio G = Hq / Hkv must be <= 32
 *   head_dim    D in {64, 128, 256}
 *   page_size   ps in {16, 32, 64, 128}
 *   capacity    C, columns of the page table (> 0); C * ps bounds seq_lens
 *
 * Allocates the workspace (work list, split partials, status word) on the
 * current device with cudaMalloc.  Returns NULL on error (pa_last_error()
 * says why: unsupported geometry, non-positive argument, CUDA failure).
 * The softmax scale defaults to 1/sqrt(head_dim).
 */
PA_API pa_plan *pa_create_plan(int batch, int heads_q, int heads_kv, int head_dim, int page_size,
                        int capacity);

/*
 * pa_run -- enqueue one attention pass on `stream`.
 *
 *   q          device, bf16 [T, Hq, D], row-major; T = cu_q_lens[B]
 *   k_pool     device, bf16 [P, ps, Hkv, D], row-major page pool of keys
 *   v_pool     device, bf16 [P, ps, Hkv, D], row-major page pool of values
 *   page_table device, int32 [B, C], row stride C; page_table[b][p] is the
 *              physical page holding keys p*ps .. p*ps+ps-1 of request b.
 *              Columns at or past ceil(seq_lens[b] / ps) are never read.
 *   seq_lens   device, int32 [B]; seq_lens[b] = KV length of request b,
 *              including this step's query tokens (0 <= seq_lens[b] <= C*ps)
 *   cu_q_lens  device, int32 [B+1], cu_q_lens[0] = 0, nondecreasing; request b
 *              owns query rows cu_q_lens[b] .. cu_q_lens[b+1]-1.  NULL means
 *              one query token per request (pure decode, T = B).
 *   out        device, bf16 [T, Hq, D]; row (t, h) = attention of query t,
 *              head h over the keys it may see (round to nearest even)
 *   lse        device, fp32 [T, Hq], natural-log log-sum-exp of the scaled
 *              scores of each row; may be NULL
 *
 * Query i (0-based within request b, q_b = cu_q_lens[b+1] - cu_q_lens[b])
 * sees keys j < seq_lens[b] - q_b + i + 1 (causal mask aligned to the end of
 * the request's KV; decode sees every key).  Query head h reads KV head
 * h / G.  All pointers must be 16-byte aligned.
 *
 * Enqueues at most five kernels (scheduler; the two-stage prefill kernel when
 * enabled, or with E4M3 pools and cu_q_lens the widening pass and the bf16
 * attention kernel over the widened requests; attention; split merge); does
 * not allocate, does not synchronise and reads no device data on the host, so
 * it can be captured in a CUDA graph.  The
 * scheduler may start while the previous pa_run on the same plan and stream
 * is still finishing (it writes the other of two work-list buffers) and ends
 * only after that run, so consecutive runs keep stream order.  Returns PA_OK, PA_ERR_INVALID
 * (NULL or misaligned pointer) or PA_ERR_CUDA (launch failure).  Problems in
 * the device-side request data are recorded in the status word instead.
 */
PA_API int pa_run(pa_plan *plan, const void *q, const void *k_pool, const void *v_pool,
           const int32_t *page_table, const int32_t *seq_lens, const int32_t *cu_q_lens,
           void *out, float *lse, pa_stream_t stream);

/* pa_destroy -- free the workspace and the plan.  NULL is a no-op.  The
 * caller must make sure no enqueued pa_run on the plan is still pending. */
PA_API void pa_destroy(pa_plan *plan);

/* Description of the last error on this thread ("" if none). */
PA_API const char *pa_last_error(void);

/* Softmax scale applied to Q K^T (finite, > 0).  Default 1/sqrt(head_dim). */
PA_API int pa_set_scale(pa_plan *plan, float scale);

/* Number of pages P in the pools (the page-pool bound, cf. the PrimTS PR's
 * "page-pool bound" of the active layer).  With P > 0 every live page id is
 * checked against [0, P) and out-of-range pages read as zeros (status bit
 * PA_STATUS_BAD_PAGE).  0 (default) trusts the table: negative ids still read
 * as zeros, but ids >= the real pool size are undefined behaviour. */
PA_API int pa_set_num_pages(pa_plan *plan, int num_pages);

/* KV splits for requests whose packed query rows fit one 128-row tile
 * (decode-like requests): 0 = automatic (default: chunks sized so that
 * the whole run is about four work items per CTA, at most
 * ceil(8 * SMs / (batch * heads_kv)) and 64 chunks per request), 1 = never
 * split, n > 1 = split every such request into min(n, its KV tiles) chunks.
 * May reallocate the workspace; call it outside graph capture. */
PA_API int pa_set_num_splits(pa_plan *plan, int num_splits);

/* Synchronise `stream`, copy the sticky status word (PA_STATUS_* bits) to
 * *status and, if clear != 0, reset it to 0.  Not capturable. */
PA_API int pa_get_status(pa_plan *plan, pa_stream_t stream, uint32_t *status, int clear);

/* Bytes of device workspace the plan holds. */
PA_API size_t pa_workspace_bytes(const pa_plan *plan);

/* Largest number of KV splits this plan can use for one request. */
PA_API int pa_max_splits(const pa_plan *plan);

/* Prefill kernel choice for head_dim 64/128.  0 (default): every query block
 * runs on the one-stage kernel (two CTAs per SM).  1: requests with two or more
 * 128-row query blocks run on the two-stage kernel, which pairs consecutive
 * blocks of one KV head so that each K/V tile feeds 256 query rows (half the
 * K/V reads) and keeps two score buffers per block.  May reallocate the
 * workspace; call it outside graph capture.  PA_ERR_UNSUPPORTED for head_dim
 * 256. */
PA_API int pa_set_two_stage_prefill(pa_plan *plan, int on);

/* Split-KV merge.  0 (default): a separate merge kernel runs after the
 * attention kernel.  1: fused -- the softmax warps of a split item write its
 * partial state, and the CTA counts itself in a per-(request, KV head)
 * counter; the CTA that arrives last merges all splits of that (request, KV
 * head) on its four softmax warps (the fused split reduction with a per-run
 * counter that "integrate PrimTS FMHA kernels", section "Planning,
 * preprocessing, and workspace ownership", names; here the scheduler zeroes
 * the counters every run and no CTA waits for another).  The fused form saves
 * the merge launch but runs each (request, KV head)'s merge on one CTA after
 * its last split, so it is slower when few (request, KV head) units carry many
 * rows and splits (0.34 against 0.28 ms per step with G = 32, D = 256, 16
 * units).  Both compute L = ln sum_s exp(L_s), O = sum_s exp(L_s - L) O_s.
 * Takes effect at the next pa_run.  PA_ERR_INVALID for a NULL plan. */
PA_API int pa_set_fused_merge(pa_plan *plan, int on);

/* Mask mode.  1 (default): causal, aligned to the end of each request's KV
 * (query i of a request with q_b tokens and kv_b keys sees keys
 * j < kv_b - q_b + i + 1).  0: every query row sees all kv_b keys of its
 * request -- the non-causal attention asked for in the review thread of
 * "Unified Triton kernel that doesn't distinguish between prefill + decode"
 * (vLLM PR #16828) for cascade attention and MLA.  Takes effect at the next
 * pa_run.  PA_ERR_INVALID for a NULL plan. */
PA_API int pa_set_causal(pa_plan *plan, int causal);

/* Row stride of page_table in int32 entries (default: capacity).  Row b of
 * the table starts at page_table + b * row_stride, so the K plane of a
 * [B, 2, C] table (K page ids in plane 0, V page field in plane 1) is passed
 * without a copy as page_table = &table[0][0][0] with row_stride = 2 * C
 * ("integrate PrimTS FMHA kernels", section "Unified page-table metadata").
 * Both K and V pages are read through these ids.  Applies to pa_run and
 * pa_append_kv.  PA_ERR_INVALID if row_stride < capacity or the plan is
 * NULL. */
PA_API int pa_set_page_table_stride(pa_plan *plan, int row_stride);

/* Decode kernel choice for runs with cu_q_lens == NULL (one query token per
 * request) and at most 32 query heads per KV head.  The decode kernel computes
 * S^T = K Q^T and O^T = V^T P^T with the 128 keys of a tile as the MMA's M
 * dimension and the G query rows (padded to 16 or 32) as N -- the same online
 * softmax ("FlashAttention", Dao et al., Algorithm 1) with 1/8 to 1/4 of the
 * tensor work of 128-row query tiles.  Default (bf16 and E4M3 pools alike):
 * head_dim 128 runs on it, head_dim 256 on the one-stage kernel.  on = 1: head_dim 128 and 256 run on
 * it.  on = 0: every such run uses the one-stage kernel.  The two paths agree
 * within the stated tolerances, not bit for bit.  Takes effect at the next
 * pa_run; no reallocation.  PA_ERR_INVALID for a NULL plan. */
PA_API int pa_set_decode_kernel(pa_plan *plan, int on);

/* Self-test of the bounded waits every kernel uses (no plan needed).  Runs
 * one CTA on the current device in which one warp waits on an mbarrier that
 * nothing arrives at, with a limit of limit_us microseconds (1 .. 1000000):
 * it gives up, sets the CTA's abort flag and PA_STATUS_TIMEOUT; a second warp
 * waiting on another such barrier with the production limit (2 s) must leave
 * through the abort flag soon after.  Writes the status word to *status_out
 * and the two waits' durations in microseconds to elapsed_us_out[0..1].
 * Synchronous (allocates 12 bytes, synchronises the device).  Returns PA_OK,
 * PA_ERR_INVALID (NULL argument, limit out of range) or PA_ERR_CUDA. */
PA_API int pa_selftest_wait_timeout(uint32_t limit_us, uint32_t *status_out,
                                    uint32_t *elapsed_us_out);

/* E4M3 (FP8) KV pools with per-tensor descales ("[Perf][FA4] Warm up dense
 * (paged) FA4 attention kernels", vLLM PR #48156: the Summary's fp8-descale
 * variants of the dense decode and prefill kernels when the KV cache is fp8,
 * and the review thread on the per-arch selector, where the fp8 kernel is
 * SM100-only and writes a bf16 output; the format is OCP FP8 E4M3: bias 7,
 * 3 mantissa bits, subnormals, S.1111.111 NaN, no infinities).  With on != 0 the k_pool and
 * v_pool of the following pa_run calls are uint8 [P, ps, Hkv, D] arrays of
 * E4M3 codes, and attention is computed as if the pools held
 * k_scale * decode(code) and v_scale * decode(code); q stays bf16, out stays
 * bf16, lse is the log-sum-exp of the descaled logits.  Decode-only runs
 * (cu_q_lens NULL) pick their kernel as for bf16 pools (pa_set_decode_kernel):
 * the E4M3 decode kernel, or the one-stage kernel's E4M3 variant; both widen
 * the codes to fp16 on chip (exact) and round q and the softmax weights P to
 * fp16 for the MMAs (q magnitudes past 65504 saturate).  Runs with cu_q_lens (prefill, chunked
 * prefill, mixed batches) take two paths in the same run:
 *   - a request with two or more query blocks (q_len > 128 / G) reads each
 *     K/V tile once per block, so its pages are widened once per run into a
 *     scratch pool of bf16 values (exact: every E4M3 value is a bf16 value)
 *     and its blocks run on the bf16 one-stage kernel, q in bf16 and P in bf16
 *     as for bf16 pools (pa_set_kv_fp8_widen sizes the scratch pool);
 *   - every other request (decode rows, short chunks) runs on the one-stage
 *     kernel's E4M3 variant, which widens each tile to fp16 on chip with q and
 *     P in fp16 as above.
 * Neither path uses the two-stage kernel (pa_set_two_stage_prefill reads bf16
 * pools only).  on = 0 restores bf16 pools (descales ignored).  Turning the
 * mode on or off resizes the plan's work-list workspace, and on allocates the
 * scratch pool of widened requests (pa_set_kv_fp8_widen; set its capacity
 * first to avoid a transient allocation), off frees it (synchronous; call it
 * outside graph capture).
 * Returns PA_ERR_INVALID for a NULL plan or a descale that is not finite and
 * > 0, PA_ERR_UNSUPPORTED for a head_dim other than 128 or 256, PA_ERR_CUDA
 * if the workspace cannot be reallocated (the plan is then unchanged). */
PA_API int pa_set_kv_fp8(pa_plan *plan, int on, float k_scale, float v_scale);

/* Scratch capacity, in pages, for widened E4M3 requests (see pa_set_kv_fp8).
 * The scratch pool holds bf16 K and V pages [max_pages, ps, Hkv, D] plus a
 * page table [B, C]; pa_set_kv_fp8 (on) allocates it, and so does this call
 * while E4M3 pools are on (cudaMalloc, synchronous: call it outside graph
 * capture; PA_ERR_CUDA if the allocation fails, after which the plan widens
 * nothing until a capacity is set that fits).  It lives until the plan is
 * destroyed, E4M3 pools are turned off or the capacity changes.  Requests of
 * two or more query blocks are widened in request order while their pages
 * (ceil(kv_len / ps) each) fit; the rest run on the E4M3 one-stage kernel, so
 * every capacity gives the same results within the stated tolerances.
 * max_pages = -1 (default): every page the batch can hold (B * C), at most
 * 512 MiB of K and V; 0: never widen; n > 0: n pages (at most B * C).  A new
 * value frees the current scratch pool first (cudaFree synchronises the
 * device).  Returns PA_ERR_INVALID for a NULL plan or max_pages < -1. */
PA_API int pa_set_kv_fp8_widen(pa_plan *plan, int max_pages);

/* Paged KV append: write this step's new K and V rows into the pools before
 * attention ("integrate PrimTS FMHA kernels", section "Planning,
 * preprocessing, and workspace ownership": the KV-cache append of the
 * preprocessing; slots per section "Unified page-table metadata").
 *   k_new, v_new   bf16 [T, Hkv, D], packed like q (row cu_q_lens[b] + i is
 *                  new token i of request b); T = cu_q_lens[B], or B when
 *                  cu_q_lens is NULL (one new token per request)
 *   k_pool, v_pool bf16 [P, ps, Hkv, D], written in place
 *   page_table, seq_lens, cu_q_lens  as for pa_run; seq_lens counts the new
 *                  tokens, so token i lands at KV position kv_b - q_b + i:
 *                  page page_table[b][j / ps], slot j % ps
 * All device pointers, 16-byte aligned, caller-owned; stream-ordered, no
 * allocation, no host synchronisation, graph-capturable.  Returns PA_OK,
 * PA_ERR_INVALID (NULL / misaligned pointer, wrong device) or PA_ERR_CUDA.
 * What cannot be placed is skipped and flagged in the plan's status word
 * (pa_get_status): a token on a page id outside [0, num_pages)
 * (PA_STATUS_BAD_PAGE; checked when pa_set_num_pages was given, negative ids
 * always), q_b > kv_b (PA_STATUS_Q_GT_KV, the request), kv_b > C * ps
 * (PA_STATUS_KV_GT_CAPACITY, the request), malformed cu_q_lens
 * (PA_STATUS_BAD_CU_Q, nothing written). */
PA_API int pa_append_kv(pa_plan *plan, const void *k_new, const void *v_new, void *k_pool,
                        void *v_pool, const int32_t *page_table, const int32_t *seq_lens,
                        const int32_t *cu_q_lens, pa_stream_t stream);

/* Kernel timing for benchmarks.  pa_profile_start makes the next `max_runs`
 * (1..4096) calls of pa_run record a CUDA event pair on their stream around
 * the attention kernel.  pa_profile_read synchronises on those events, writes
 * the summed attention-kernel time in milliseconds, the number of runs
 * recorded and the number of kernels each pa_run launches, and turns the
 * recording off.  While recording, pa_run must not be captured in a graph.
 * The events are owned by the plan. */
PA_API int pa_profile_start(pa_plan *plan, int max_runs);
PA_API int pa_profile_read(pa_plan *plan, float *attn_ms, int *n_runs, int *launches_per_run);

/*
 * pa_run_noalloc -- the same attention pass as pa_run, for callers that cannot
 * allocate device memory.  (The source pages have no counterpart: this entry
 * point exists for integration, not for the method.)
 *
 * Some callers cannot call cudaMalloc at the point where they run attention:
 * an engine whose device memory is fully budgeted by its own allocator (a raw
 * cudaMalloc would bypass its accounting and can fail late, or take memory
 * the engine has promised elsewhere), or a serving loop where a synchronous
 * allocation would stall the device.  pa_create_plan allocates a workspace,
 * so such callers use this entry point instead: no plan, no cudaMalloc, no
 * cudaFree, no allocating library routine.  The caller still passes every
 * input and output.
 *
 * Scratch: the work list and the status word live in one file-scope device
 * array of PA_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU which loads the
 * library holds until the process exits.  A geometry whose worst-case work
 * list does not fit (batch * heads_kv * ceil(capacity * page_size * G / 128)
 * items of 32 bytes, plus 44 bytes per request and a small header) is
 * rejected with PA_ERR_UNSUPPORTED and a message saying so.  KV splitting is
 * not used on this path (each (request, KV head, query block) is one item),
 * so there is no split merge and no partial-state storage.  The pools are
 * bf16 only: nothing in the arguments says whether they hold E4M3 codes, so
 * an fp8 pool passed here would be read as bf16 without an error.
 *
 * All calls share the array and it keeps the last call's contents; each call
 * clears the header it relies on (status word, item count) on `stream` before
 * its kernels run.  Calls whose work overlaps on the GPU (different streams,
 * or several threads) race on the array and must be serialised by the caller.
 *
 * The first call on a device performs a one-time set-up on that device with
 * synchronous runtime calls (it resolves the array's device address with
 * cudaGetSymbolAddress and sets the kernel's shared-memory limit).  Later
 * calls only enqueue work.
 *
 * Arguments are those of pa_create_plan followed by those of pa_run, plus
 *   num_pages  pool size P for page-id checks (0 = trust the table)
 *   scale      softmax scale (> 0), or 0 for 1/sqrt(head_dim)
 * Returns PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED or PA_ERR_CUDA.  Bad
 * request data found on the device (PA_STATUS_* bits, as for pa_run) is
 * recorded in the array's status word: read it with pa_noalloc_get_status
 * before the next pa_run_noalloc on the device, which clears it.
 */
#define PA_NOALLOC_SCRATCH_BYTES (8u << 20)
PA_API int pa_run_noalloc(int batch, int heads_q, int heads_kv, int head_dim, int page_size,
                          int capacity, int num_pages, float scale, const void *q,
                          const void *k_pool, const void *v_pool, const int32_t *page_table,
                          const int32_t *seq_lens, const int32_t *cu_q_lens, void *out,
                          float *lse, pa_stream_t stream);

/* Status word of the last pa_run_noalloc on the current device (no paper
 * counterpart either): synchronises `stream`, copies the PA_STATUS_* bits to
 * *status and, if clear != 0, resets them.  Allocates nothing.  Must be read
 * before the next pa_run_noalloc on the device, which clears the word.
 * Returns PA_OK, PA_ERR_INVALID (NULL status) or PA_ERR_CUDA. */
PA_API int pa_noalloc_get_status(pa_stream_t stream, uint32_t *status, int clear);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
