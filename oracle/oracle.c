/*
 * Paged-KV grouped-query attention: plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link or call this file.  Only the
 * tests, the package's build-and-smoke entry and the CPU baseline of the
 * benchmark use it.  It shares no code, header, table or helper with the
 * CUDA path.
 *
 * What it computes, for every request b, query head h and query token i:
 *
 *     O[t, h, :] = softmax_j( scale * q[t,h,:] . K_b[j, g, :] ) V_b[j, g, :]
 *     LSE[t, h]  = ln sum_j exp( scale * q[t,h,:] . K_b[j, g, :] )
 *
 * over the keys j that query i may see.  Sources, by topic:
 *
 *  - Page resolution.  "integrate PrimTS FMHA kernels" (TensorRT-LLM PR
 *    #17399), section "Unified page-table metadata": the page table is an
 *    int32 row-strided [B, C] array plus live int32 seq_lens[B]; logical
 *    page p of request b is block_tables[b, p]; seq_lens[b] fixes how many
 *    pages are live, so capacity columns past it are never consumed.  Here
 *    key j of request b sits in physical page table[b][j / ps], slot j % ps,
 *    and no column at or past ceil(seq_lens[b] / ps) is ever read.
 *  - Varlen packed queries and GQA.  "Unified Triton kernel that doesn't
 *    distinguish between prefill + decode" (vLLM PR #16828), description:
 *    queries are packed like flash_attn_varlen_func (cu_q_lens offsets) and
 *    one kernel handles any query length.  Query head h reads KV head
 *    h / (Hq / Hkv) (consecutive groups; the pages do not fix the map, this
 *    is the flash-attention convention).
 *  - Causal mask by select.  Same vLLM PR, review thread on the kernel:
 *    scores outside the mask are replaced by -inf with a select, not an add.
 *    The mask is aligned to the end of the request's KV: with
 *    q_b = cu[b+1]-cu[b] and kv_b = seq_lens[b], query i (0-based within
 *    the request) sees keys j < kv_b - q_b + i + 1.  For decode (q_b = 1)
 *    that is every key.
 *  - seq_lens is the whole KV length including this step's tokens
 *    (PrimTS PR, "Unified page-table metadata": context reads
 *    sequence_lengths directly).
 *  - LSE is the natural-log log-sum-exp of the scaled scores (the pages
 *    never define it; flash-attention convention).
 *  - A query row that sees no key (only possible for invalid input with
 *    q_b > kv_b) gets O = 0 and LSE = -inf.
 *
 * Inputs are bf16 bit patterns, widened exactly to double.  All arithmetic
 * is fp64, one (token, head) row at a time: the scores of the row, their
 * maximum, the exponentials, their sum, then the weighted sum of V.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double: the bf16 bits are the high half of an IEEE binary32. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    int B, Hq, Hkv, D, ps, C, num_pages;
    const uint16_t *q, *k_pool, *v_pool;
    const int32_t *page_table, *seq_lens, *cu_q_lens;
    double scale;
    int non_causal;       /* 0: causal mask (default); 1: every row sees all kv_b keys */
    /* fp8 pools: when k8 is set, K and V are e4m3 codes [P, ps, Hkv, D] and
     * the values are code * k_scale, code * v_scale */
    const uint8_t *k8, *v8;
    double k_scale, v_scale;
    double *out, *lse;
    /* rows to compute: either all (rows == NULL) or a list of (t, h) */
    const int32_t *row_t, *row_h;
    long n_rows;
    /* request index of each token */
    const int32_t *tok_req;
    /* work distribution */
    long next;
    pthread_mutex_t lock;
    int error;
} job_t;

/* Element (page, slot, kv head, d) of a pool laid out [P, ps, Hkv, D]. */
static double pool_at(const job_t *J, const uint16_t *pool, long page, long slot, long g, long d) {
    long idx = ((page * J->ps + slot) * J->Hkv + g) * J->D + d;
    return bf16_to_double(pool[idx]);
}

/*
 * FP8 E4M3 code -> double, from the format's definition (the OCP 8-bit
 * floating point format, E4M3 variant): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 encodes subnormals m * 2^-9; the one
 * pattern S.1111.111 is NaN and there are no infinities (largest 448).
 */
static double e4m3_to_double(uint8_t c) {
    const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = m * ldexp(1.0, -9);
    else v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return sgn ? -v : v;
}

static double k_at(const job_t *J, long page, long slot, long g, long d) {
    if (J->k8) return J->k_scale * e4m3_to_double(J->k8[((page * J->ps + slot) * J->Hkv + g) * J->D + d]);
    return pool_at(J, J->k_pool, page, slot, g, d);
}

static double v_at(const job_t *J, long page, long slot, long g, long d) {
    if (J->v8) return J->v_scale * e4m3_to_double(J->v8[((page * J->ps + slot) * J->Hkv + g) * J->D + d]);
    return pool_at(J, J->v_pool, page, slot, g, d);
}

/* One output row: token t (global packed index), query head h.  Returns 0 or
 * an error code (1 = page id outside the pool inside the live range). */
static int one_row(const job_t *J, long t, int h, double *o_row, double *lse_out,
                   double *s /* scratch, kv_b doubles */) {
    const int b = J->tok_req[t];
    const long q0 = J->cu_q_lens ? J->cu_q_lens[b] : b;
    const long q_b = J->cu_q_lens ? (J->cu_q_lens[b + 1] - J->cu_q_lens[b]) : 1;
    const long kv_b = J->seq_lens[b];
    const long i = t - q0;                 /* query position within the request */
    const int G = J->Hq / J->Hkv;
    const int g = h / G;                   /* KV head read by query head h */
    const int D = J->D;

    /* visible keys: j < n, with the causal limit aligned to the end of KV */
    long n = kv_b - q_b + i + 1;
    if (J->non_causal) n = kv_b;           /* non-causal: every key of the request */
    if (n > kv_b) n = kv_b;
    if (n < 0) n = 0;

    for (int d = 0; d < D; ++d) o_row[d] = 0.0;
    if (n == 0) {
        *lse_out = -INFINITY;
        return 0;
    }

    const uint16_t *qrow = J->q + ((long)t * J->Hq + h) * D;
    double m = -INFINITY;
    for (long j = 0; j < n; ++j) {
        long page = J->page_table[(long)b * J->C + j / J->ps];
        if (page < 0 || (J->num_pages > 0 && page >= J->num_pages)) return 1;
        long slot = j % J->ps;
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += bf16_to_double(qrow[d]) * k_at(J, page, slot, g, d);
        s[j] = J->scale * acc;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (long j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (long j = 0; j < n; ++j) {
        long page = J->page_table[(long)b * J->C + j / J->ps];
        long slot = j % J->ps;
        double w = s[j] / l;
        for (int d = 0; d < D; ++d) o_row[d] += w * v_at(J, page, slot, g, d);
    }
    *lse_out = m + log(l);
    return 0;
}

static long total_tokens(const job_t *J) {
    return J->cu_q_lens ? J->cu_q_lens[J->B] : J->B;
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    long max_kv = 1;
    for (int b = 0; b < J->B; ++b)
        if (J->seq_lens[b] > max_kv) max_kv = J->seq_lens[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)max_kv);
    if (!s) {
        pthread_mutex_lock(&J->lock);
        J->error = 2;
        pthread_mutex_unlock(&J->lock);
        return NULL;
    }
    const long n_units = J->row_t ? J->n_rows : total_tokens(J) * J->Hq;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        long u = J->next++;
        int stop = J->error != 0;
        pthread_mutex_unlock(&J->lock);
        if (u >= n_units || stop) break;
        long t;
        int h;
        double *o, *l;
        if (J->row_t) {
            t = J->row_t[u];
            h = J->row_h[u];
            o = J->out + u * J->D;
            l = J->lse + u;
        } else {
            t = u / J->Hq;
            h = (int)(u % J->Hq);
            o = J->out + u * J->D;
            l = J->lse + u;
        }
        int rc = one_row(J, t, h, o, l, s);
        if (rc) {
            pthread_mutex_lock(&J->lock);
            if (!J->error) J->error = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    free(s);
    return NULL;
}

static int run_job(job_t *J, int nthreads) {
    long T = total_tokens(J);
    int32_t *tok_req = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    if (!tok_req) return 2;
    for (int b = 0; b < J->B; ++b) {
        long a = J->cu_q_lens ? J->cu_q_lens[b] : b;
        long e = J->cu_q_lens ? J->cu_q_lens[b + 1] : b + 1;
        for (long t = a; t < e; ++t) tok_req[t] = b;
    }
    J->tok_req = tok_req;
    J->next = 0;
    J->error = 0;
    pthread_mutex_init(&J->lock, NULL);
    if (nthreads < 1) nthreads = 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J->lock);
    free(th);
    free(tok_req);
    return J->error;
}

/* Every (token, head) row.  out: [T, Hq, D] doubles, lse: [T, Hq] doubles.
 * cu_q_lens may be NULL (one query token per request).  num_pages <= 0
 * disables the page-id bound check (ids must still be >= 0).
 * Returns 0, 1 (a live page id is out of range) or 2 (out of memory). */
int oracle_paged_attention(int B, int Hq, int Hkv, int D, int ps, int C, int num_pages,
                           const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                           const int32_t *page_table, const int32_t *seq_lens,
                           const int32_t *cu_q_lens, double scale, double *out, double *lse,
                           int nthreads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.ps = ps; J.C = C; J.num_pages = num_pages;
    J.q = q; J.k_pool = k_pool; J.v_pool = v_pool;
    J.page_table = page_table; J.seq_lens = seq_lens; J.cu_q_lens = cu_q_lens;
    J.scale = scale; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}

/*
 * The same with a mask mode.  causal = 0 drops the causal limit: every query
 * row of request b sees all kv_b keys.  "Unified Triton kernel that doesn't
 * distinguish between prefill + decode" (vLLM PR #16828), review thread on the
 * masking: non-causal attention is asked for (cascade attention, MLA); the
 * plainest reading is the same softmax over the request's whole KV.
 */
int oracle_paged_attention_mode(int B, int Hq, int Hkv, int D, int ps, int C, int num_pages,
                                const uint16_t *q, const uint16_t *k_pool,
                                const uint16_t *v_pool, const int32_t *page_table,
                                const int32_t *seq_lens, const int32_t *cu_q_lens, double scale,
                                int causal, double *out, double *lse, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.ps = ps; J.C = C; J.num_pages = num_pages;
    J.q = q; J.k_pool = k_pool; J.v_pool = v_pool;
    J.page_table = page_table; J.seq_lens = seq_lens; J.cu_q_lens = cu_q_lens;
    J.scale = scale; J.out = out; J.lse = lse;
    J.non_causal = causal ? 0 : 1;
    return run_job(&J, nthreads);
}

/*
 * FP8 KV cache with per-tensor descales (the "fp8 KV cache with descale,
 * bf16 output" variants that "[Perf][FA4] Warm up dense (paged) FA4 attention
 * kernels", vLLM PR #48156, warms up): k8 / v8 are E4M3 codes laid out like
 * the bf16 pools and K = code * k_scale, V = code * v_scale.  q stays bf16;
 * everything else is the causal attention above, in fp64.
 */
int oracle_paged_attention_fp8(int B, int Hq, int Hkv, int D, int ps, int C, int num_pages,
                               const uint16_t *q, const uint8_t *k8, const uint8_t *v8,
                               double k_scale, double v_scale, const int32_t *page_table,
                               const int32_t *seq_lens, const int32_t *cu_q_lens, double scale,
                               double *out, double *lse, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.ps = ps; J.C = C; J.num_pages = num_pages;
    J.q = q; J.k8 = k8; J.v8 = v8; J.k_scale = k_scale; J.v_scale = v_scale;
    J.page_table = page_table; J.seq_lens = seq_lens; J.cu_q_lens = cu_q_lens;
    J.scale = scale; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}

/* E4M3 decoding of n codes (exposed for the pins). */
void oracle_e4m3_decode(const uint8_t *codes, long n, double *out) {
    for (long i = 0; i < n; ++i) out[i] = e4m3_to_double(codes[i]);
}

/* Only the listed rows: row u is (token row_t[u], head row_h[u]); out is
 * [n_rows, D], lse is [n_rows].  Same return codes. */
int oracle_paged_attention_rows(int B, int Hq, int Hkv, int D, int ps, int C, int num_pages,
                                const uint16_t *q, const uint16_t *k_pool,
                                const uint16_t *v_pool, const int32_t *page_table,
                                const int32_t *seq_lens, const int32_t *cu_q_lens, double scale,
                                const int32_t *row_t, const int32_t *row_h, long n_rows,
                                double *out, double *lse, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.ps = ps; J.C = C; J.num_pages = num_pages;
    J.q = q; J.k_pool = k_pool; J.v_pool = v_pool;
    J.page_table = page_table; J.seq_lens = seq_lens; J.cu_q_lens = cu_q_lens;
    J.scale = scale; J.out = out; J.lse = lse;
    J.row_t = row_t; J.row_h = row_h; J.n_rows = n_rows;
    return run_job(&J, nthreads);
}

/*
 * Merge of partial attention states computed over disjoint key ranges
 * (split-KV decode with a log-sum-exp merge).  The PrimTS PR ("Planning,
 * preprocessing, and workspace ownership") and the FA4 warm-up PR (review
 * thread on is_split_kv) name the split-KV reduction without spelling it
 * out; this is the exact identity it rests on.  For one row with n partial
 * states (O_s normalised over its own keys, L_s its log-sum-exp):
 *     L = ln sum_s exp(L_s),   O = sum_s exp(L_s - L) O_s.
 * A state with L_s = -inf (it saw no key) has weight 0; if every state is
 * empty the row is O = 0, L = -inf.
 * o_s: [n, D], lse_s: [n]; o: [D], lse: [1].
 */
void oracle_merge_states(int n, int D, const double *o_s, const double *lse_s, double *o,
                         double *lse) {
    double m = -INFINITY;
    for (int s = 0; s < n; ++s)
        if (lse_s[s] > m) m = lse_s[s];
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int s = 0; s < n; ++s) sum += exp(lse_s[s] - m);
    double L = m + log(sum);
    for (int s = 0; s < n; ++s) {
        double w = exp(lse_s[s] - L);
        for (int d = 0; d < D; ++d) o[d] += w * o_s[(long)s * D + d];
    }
    *lse = L;
}

/*
 * Paged KV append: the step before attention in serving, which writes this
 * step's new K and V rows into the page pool.  "integrate PrimTS FMHA
 * kernels" (TensorRT-LLM PR #17399), section "Planning, preprocessing, and
 * workspace ownership", reuses the engine's fused preprocessing for the
 * KV-cache append; the slot a token lands in follows section "Unified
 * page-table metadata": logical page p of request b is page_table[b][p], and
 * seq_lens[b] counts this step's tokens.  So with q_b = cu[b+1] - cu[b] new
 * tokens (q_b = 1 when cu_q_lens is NULL) and kv_b = seq_lens[b], new token i
 * of request b (packed row t = cu[b] + i of k_new / v_new, [T, Hkv, D]) is KV
 * position j = kv_b - q_b + i and is copied, all Hkv heads at once, to
 * page page_table[b][j / ps], slot j % ps of k_pool / v_pool ([P, ps, Hkv, D]).
 * Nothing else in the pools changes.
 *
 * What cannot be placed is skipped and reported in the returned bit mask
 * (the same bits as the CUDA path's status word); the pages fix no policy,
 * this reading skips the least:
 *   1  a token whose page id is outside [0, num_pages) (checked when
 *      num_pages > 0; negative ids always): that token only
 *   2  q_b > kv_b: the whole request
 *   4  kv_b > C * ps: the whole request
 *   8  malformed cu_q_lens (cu[0] != 0, decreasing, or a total past
 *      B * C * ps): nothing is written
 */
int oracle_append_kv(int B, int Hkv, int D, int ps, int C, int num_pages,
                     const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_pool,
                     uint16_t *v_pool, const int32_t *page_table, const int32_t *seq_lens,
                     const int32_t *cu_q_lens) {
    int flags = 0;
    const long row = (long)Hkv * D;   /* elements of one token's K (or V) row */
    if (cu_q_lens) {
        /* a total past B * C * ps cannot come from valid requests (q_b <= kv_b
         * <= C * ps), so it is treated as malformed too */
        if (cu_q_lens[0] != 0 || (long)cu_q_lens[B] > (long)B * C * ps) return 8;
        for (int b = 0; b < B; ++b)
            if (cu_q_lens[b + 1] < cu_q_lens[b]) return 8;
    }
    for (int b = 0; b < B; ++b) {
        const long t0 = cu_q_lens ? cu_q_lens[b] : b;
        const int qb = cu_q_lens ? cu_q_lens[b + 1] - cu_q_lens[b] : 1;
        const int kv = seq_lens[b];
        if (qb == 0) continue;
        if (qb > kv) { flags |= 2; continue; }
        if ((long)kv > (long)C * ps) { flags |= 4; continue; }
        for (int i = 0; i < qb; ++i) {
            const int j = kv - qb + i;
            const long page = page_table[(long)b * C + j / ps];
            if (page < 0 || (num_pages > 0 && page >= num_pages)) { flags |= 1; continue; }
            const long dst = (page * ps + j % ps) * row;
            const long src = (t0 + i) * row;
            for (long e = 0; e < row; ++e) {
                k_pool[dst + e] = k_new[src + e];
                v_pool[dst + e] = v_new[src + e];
            }
        }
    }
    return flags;
}
