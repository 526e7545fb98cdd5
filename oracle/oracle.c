/*
 * Plain fp64 CPU oracle for exact attention and its split-KV decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load or call this
 * library: only the test suite, the package's smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only at the seeded bf16 inputs.
 *
 * What is computed (the plain definition the tiled method must reproduce):
 *   "FlashAttention in Ascend CANN ops-transformer" (ai6s.net), section 二,
 *   step 2: the block-by-block online softmax gives a result identical to
 *   standard attention; section 四 fixes the [batch, seq_len, num_heads,
 *   head_dim] layout and softmax_scale; section 五 fixes the causal flag (keys
 *   after the query take no part in the softmax) and head_dim 64/128/256.
 *   "FlashAttention-2 (TH)" (systems-analysis.info): exact, no approximation.
 *
 *   For batch b, query head h, key/value head g = h / (Hq/Hkv), query row i:
 *     s_j   = scale * sum_d q[b,i,h,d] * k[b,j,g,d]          for allowed j
 *     allowed(i,j) = j < Lk  and  (not causal  or  j <= i + (Lk - Lq))
 *     m     = max_j s_j
 *     O_i   = sum_j exp(s_j - m) v[b,j,g,:] / sum_j exp(s_j - m)
 *     L_i   = m + ln sum_j exp(s_j - m)      (natural-log log-sum-exp)
 *   Masked scores are -infinity (additive mask), so they contribute exp = 0.
 *
 * Inputs are bf16 bit patterns (uint16); each converts exactly to fp64.
 * All arithmetic is fp64.  Work is spread over rows with POSIX threads; each
 * row is computed independently and in a fixed order, so results do not
 * depend on the thread count.
 *
 * Functions (all return 0 on success, nonzero on a bad argument):
 *   oracle_attention_rows   - the definition above, for a list of rows.
 *   oracle_probs            - the full probability matrix (small inputs).
 *   oracle_online_rows      - the pages' tiled algorithm (blocks of keys,
 *                             running max and sum, blockwise O/L), in fp64.
 *   oracle_lse_merge        - merge of per-chunk (O_c, L_c) through their
 *                             log-sum-exp, the split-KV combine rule.
 *   oracle_decode_rows      - one query token against a KV cache with
 *                             per-sequence lengths (the definition, Lq = 1).
 *   oracle_decode_split_rows- the same, computed chunk by chunk and merged.
 *   oracle_attention_varlen_rows - a packed batch of variable-length
 *                             sequences (block-diagonal attention, the
 *                             "block diagonal" bias of the xformers page):
 *                             the definition per sequence; a row with no
 *                             allowed key gets O = 0 and L = -inf.
 *   oracle_quantize_kv_int8 - symmetric int8 quantisation of K/V rows with
 *                             one fp32 scale per (sequence, token, head), in
 *                             the exact fp32 steps the kernels take.
 *   oracle_decode_int8_rows - decode against an int8 cache (the MNN
 *                             attention_mode page's KV-INT8: K int8 with V
 *                             unquantised, or K and V int8): the cache is
 *                             dequantised exactly in fp64, then the
 *                             definition.
 *   oracle_attention_backward - gradients dQ, dK, dV of the forward for an
 *                             upstream gradient dO (the backward pass the
 *                             xformers page pairs with every forward op, and
 *                             the training use the FlashAttention-2 page
 *                             reports): P of the definition, dV = P^T dO,
 *                             dP = dO V^T, dS = P o (dP - rowsum(dO o O)),
 *                             dQ = scale dS K, dK = scale dS^T Q; GQA heads
 *                             sum into their K/V head.
 *   oracle_e4m3_decode / oracle_e4m3_encode - the OCP 8-bit float e4m3
 *                             (1 sign, 4 exponent bits with bias 7, 3 mantissa
 *                             bits, subnormals at exponent field 0, no
 *                             infinities, S.1111.111 = NaN, largest finite
 *                             448), written from that definition; encoding
 *                             rounds to nearest even and saturates at +-448.
 *   oracle_quantize_fp8     - per-(batch, head) e4m3 quantisation of a bf16
 *                             tensor (the FP8 inputs of FlashAttention-3, named
 *                             on the FlashAttention-2 page): amax over the
 *                             head's L x D slice, inv = 448 / amax and
 *                             descale = amax / 448 in fp32, code =
 *                             e4m3(x * inv) with the product in fp32; both
 *                             factors are 1 when amax < 2^-110.
 *   oracle_attention_fp8_rows - the definition above on e4m3 inputs: every
 *                             operand is code * descale (its head's factor),
 *                             dequantised exactly in fp64.
 *   oracle_decode_paged_rows- one query token against a paged cache: key j
 *                             of sequence b is row j % page_size of page
 *                             block_table[b][j / page_size] ("paged" is one of
 *                             the structured attention-bias layouts listed on
 *                             the xformers page); the definition over the
 *                             keys gathered in order.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* Thread pool over an index range.                                          */
/* ------------------------------------------------------------------------- */
typedef void (*row_fn)(void* ctx, int64_t r, double* scratch);

typedef struct {
    row_fn fn;
    void* ctx;
    int64_t begin, end;
    size_t scratch_len;
    int failed;
} worker_arg;

static void* worker_main(void* p) {
    worker_arg* a = (worker_arg*)p;
    double* scratch = NULL;
    if (a->scratch_len) {
        scratch = (double*)malloc(a->scratch_len * sizeof(double));
        if (!scratch) { a->failed = 1; return NULL; }
    }
    for (int64_t r = a->begin; r < a->end; ++r) a->fn(a->ctx, r, scratch);
    free(scratch);
    return NULL;
}

static int parallel_rows(row_fn fn, void* ctx, int64_t n, size_t scratch_len, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    if ((int64_t)nthreads > n) nthreads = (int)(n > 0 ? n : 1);
    pthread_t th[512];
    worker_arg args[512];
    int64_t chunk = (n + nthreads - 1) / nthreads;
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        int64_t b = (int64_t)t * chunk, e = b + chunk;
        if (b > n) b = n;
        if (e > n) e = n;
        args[t] = (worker_arg){fn, ctx, b, e, scratch_len, 0};
    }
    if (nthreads == 1) {
        worker_main(&args[0]);
        return args[0].failed;
    }
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, worker_main, &args[t]) != 0) { rc = 1; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    for (int t = 0; t < started; ++t) rc |= args[t].failed;
    return rc;
}

/* ------------------------------------------------------------------------- */
/* The definition, one query row.                                            */
/* ------------------------------------------------------------------------- */
/* q_row: D values; k0/v0: key 0 of this (b, g); key j sits at +j*kv_stride.
 * n_keys: Lk; limit: keys j <= limit are allowed (limit >= n_keys-1 means no
 * causal cut).  s: scratch of n_keys doubles.  Writes D outputs and the LSE. */
static void attend_one_row(const uint16_t* q_row, const uint16_t* k0, const uint16_t* v0,
                           int64_t kv_stride, int64_t n_keys, int64_t limit, int D,
                           double scale, double* o, double* lse, double* s) {
    double m = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
        if (j > limit) { s[j] = -INFINITY; continue; }      /* additive -inf mask */
        const uint16_t* kr = k0 + j * kv_stride;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(kr[d]);
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        if (s[j] == -INFINITY) continue;                     /* exp(-inf) = 0 */
        double p = exp(s[j] - m);
        sum += p;
        const uint16_t* vr = v0 + j * kv_stride;
        for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_double(vr[d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= sum;
    *lse = m + log(sum);
}

typedef struct {
    const uint16_t *q, *k, *v;
    int B, Lq, Lk, Hq, Hkv, D, causal;
    double scale;
    const int64_t* rows;
    double *o, *lse;
    int64_t block;    /* online variant: keys per block */
} attn_ctx;

/* Decode a flat row index (b*Hq + h)*Lq + i. */
static void split_row(const attn_ctx* c, int64_t flat, int* b, int* h, int64_t* i) {
    *i = flat % c->Lq;
    int64_t bh = flat / c->Lq;
    *h = (int)(bh % c->Hq);
    *b = (int)(bh / c->Hq);
}

static void attn_row_task(void* vctx, int64_t r, double* scratch) {
    const attn_ctx* c = (const attn_ctx*)vctx;
    int b, h;
    int64_t i;
    split_row(c, c->rows[r], &b, &h, &i);
    int group = c->Hq / c->Hkv;
    int g = h / group;
    const uint16_t* q_row = c->q + (((int64_t)b * c->Lq + i) * c->Hq + h) * c->D;
    const uint16_t* k0 = c->k + ((int64_t)b * c->Lk * c->Hkv + g) * c->D;
    const uint16_t* v0 = c->v + ((int64_t)b * c->Lk * c->Hkv + g) * c->D;
    int64_t limit = c->causal ? i + (int64_t)(c->Lk - c->Lq) : (int64_t)c->Lk - 1;
    attend_one_row(q_row, k0, v0, (int64_t)c->Hkv * c->D, c->Lk, limit, c->D, c->scale,
                   c->o + r * c->D, c->lse + r, scratch);
}

static int check_shape(int B, int Lq, int Lk, int Hq, int Hkv, int D, int causal) {
    if (B <= 0 || Lq <= 0 || Lk <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return 1;
    if (Hq % Hkv) return 1;
    if (causal && Lq > Lk) return 1;   /* a query row would have no key */
    return 0;
}

/* q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D] bf16 bits; rows: flat (b*Hq+h)*Lq+i;
 * o [nrows, D], lse [nrows]. */
int oracle_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          int B, int Lq, int Lk, int Hq, int Hkv, int D,
                          double scale, int causal,
                          const int64_t* rows, int64_t nrows,
                          double* o, double* lse, int nthreads) {
    if (check_shape(B, Lq, Lk, Hq, Hkv, D, causal)) return 1;
    int64_t total = (int64_t)B * Hq * Lq;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return 2;
    attn_ctx c = {q, k, v, B, Lq, Lk, Hq, Hkv, D, causal, scale, rows, o, lse, 0};
    return parallel_rows(attn_row_task, &c, nrows, (size_t)Lk, nthreads);
}

/* Probability matrix P [B,Hq,Lq,Lk] of the definition (small inputs only). */
int oracle_probs(const uint16_t* q, const uint16_t* k, int B, int Lq, int Lk, int Hq,
                 int Hkv, int D, double scale, int causal, double* p) {
    if (check_shape(B, Lq, Lk, Hq, Hkv, D, causal)) return 1;
    int group = Hq / Hkv;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h)
            for (int64_t i = 0; i < Lq; ++i) {
                double* row = p + (((int64_t)b * Hq + h) * Lq + i) * Lk;
                const uint16_t* q_row = q + (((int64_t)b * Lq + i) * Hq + h) * D;
                int64_t limit = causal ? i + (int64_t)(Lk - Lq) : (int64_t)Lk - 1;
                double m = -INFINITY;
                for (int64_t j = 0; j < Lk; ++j) {
                    if (j > limit) { row[j] = -INFINITY; continue; }
                    const uint16_t* kr = k + (((int64_t)b * Lk + j) * Hkv + h / group) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(kr[d]);
                    row[j] = scale * dot;
                    if (row[j] > m) m = row[j];
                }
                double sum = 0.0;
                for (int64_t j = 0; j < Lk; ++j) {
                    row[j] = (row[j] == -INFINITY) ? 0.0 : exp(row[j] - m);
                    sum += row[j];
                }
                for (int64_t j = 0; j < Lk; ++j) row[j] /= sum;
            }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* The pages' tiled algorithm, in fp64 (section 二 of the ops-transformer     */
/* page: 1. cut K/V into blocks; 2. per block, update the running max and    */
/* running sum; 3. accumulate O and L block by block).                       */
/* ------------------------------------------------------------------------- */
static void online_row_task(void* vctx, int64_t r, double* acc) {
    const attn_ctx* c = (const attn_ctx*)vctx;
    int b, h;
    int64_t i;
    split_row(c, c->rows[r], &b, &h, &i);
    int D = c->D, g = h / (c->Hq / c->Hkv);
    const uint16_t* q_row = c->q + (((int64_t)b * c->Lq + i) * c->Hq + h) * D;
    int64_t stride = (int64_t)c->Hkv * D;
    const uint16_t* k0 = c->k + ((int64_t)b * c->Lk * c->Hkv + g) * D;
    const uint16_t* v0 = c->v + ((int64_t)b * c->Lk * c->Hkv + g) * D;
    int64_t limit = c->causal ? i + (int64_t)(c->Lk - c->Lq) : (int64_t)c->Lk - 1;

    double m = -INFINITY, l = 0.0;           /* running max, running sum */
    for (int d = 0; d < D; ++d) acc[d] = 0.0; /* unnormalised output     */
    double* sblk = acc + D;                  /* scores of one block     */
    for (int64_t j0 = 0; j0 < c->Lk; j0 += c->block) {
        int64_t j1 = j0 + c->block < c->Lk ? j0 + c->block : c->Lk;
        /* scores of this block, masked ones at -inf */
        double bmax = -INFINITY;
        for (int64_t j = j0; j < j1; ++j) {
            double s = -INFINITY;
            if (j <= limit) {
                double dot = 0.0;
                const uint16_t* kr = k0 + j * stride;
                for (int d = 0; d < D; ++d) dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(kr[d]);
                s = c->scale * dot;
            }
            sblk[j - j0] = s;
            if (s > bmax) bmax = s;
        }
        if (bmax == -INFINITY) continue;     /* block fully masked: nothing changes */
        double m_new = m > bmax ? m : bmax;
        double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
        l *= alpha;
        for (int d = 0; d < D; ++d) acc[d] *= alpha;
        for (int64_t j = j0; j < j1; ++j) {
            double s = sblk[j - j0];
            if (s == -INFINITY) continue;
            double p = exp(s - m_new);
            l += p;
            const uint16_t* vr = v0 + j * stride;
            for (int d = 0; d < D; ++d) acc[d] += p * bf16_bits_to_double(vr[d]);
        }
        m = m_new;
    }
    for (int d = 0; d < D; ++d) c->o[r * D + d] = acc[d] / l;
    c->lse[r] = m + log(l);
}

int oracle_online_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       int B, int Lq, int Lk, int Hq, int Hkv, int D,
                       double scale, int causal, int64_t block,
                       const int64_t* rows, int64_t nrows,
                       double* o, double* lse, int nthreads) {
    if (check_shape(B, Lq, Lk, Hq, Hkv, D, causal) || block <= 0) return 1;
    int64_t total = (int64_t)B * Hq * Lq;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return 2;
    attn_ctx c = {q, k, v, B, Lq, Lk, Hq, Hkv, D, causal, scale, rows, o, lse, block};
    return parallel_rows(online_row_task, &c, nrows, (size_t)D + (size_t)block, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Split-KV combine: chunk results (O_c normalised, L_c natural-log LSE)     */
/* merge into L = log sum_c exp(L_c), O = sum_c exp(L_c - L) O_c.  An empty  */
/* chunk has L_c = -inf and weight 0.                                        */
/* ------------------------------------------------------------------------- */
int oracle_lse_merge(const double* o_parts, const double* l_parts, int S, int D,
                     double* o, double* lse) {
    if (S <= 0 || D <= 0) return 1;
    double m = -INFINITY;
    for (int c = 0; c < S; ++c) if (l_parts[c] > m) m = l_parts[c];
    if (m == -INFINITY) return 3;            /* no key at all */
    double sum = 0.0;
    for (int c = 0; c < S; ++c) sum += (l_parts[c] == -INFINITY) ? 0.0 : exp(l_parts[c] - m);
    double L = m + log(sum);
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int c = 0; c < S; ++c) {
        if (l_parts[c] == -INFINITY) continue;
        double w = exp(l_parts[c] - L);
        for (int d = 0; d < D; ++d) o[d] += w * o_parts[(int64_t)c * D + d];
    }
    *lse = L;
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Decode: one query token per sequence against a KV cache.                  */
/* q [B,1,Hq,D]; caches [B,Lmax,Hkv,D]; seqlens[b] keys of sequence b count. */
/* rows: flat b*Hq + h.                                                      */
/* ------------------------------------------------------------------------- */
typedef struct {
    const uint16_t *q, *kc, *vc;
    const int32_t* seqlens;
    int B, Hq, Hkv, D, Lmax, S;
    double scale;
    const int64_t* rows;
    double *o, *lse;
} dec_ctx;

static void decode_row_task(void* vctx, int64_t r, double* scratch) {
    const dec_ctx* c = (const dec_ctx*)vctx;
    int64_t flat = c->rows[r];
    int h = (int)(flat % c->Hq), b = (int)(flat / c->Hq);
    int g = h / (c->Hq / c->Hkv);
    int64_t n = c->seqlens[b];
    const uint16_t* q_row = c->q + ((int64_t)b * c->Hq + h) * c->D;
    const uint16_t* k0 = c->kc + ((int64_t)b * c->Lmax * c->Hkv + g) * c->D;
    const uint16_t* v0 = c->vc + ((int64_t)b * c->Lmax * c->Hkv + g) * c->D;
    attend_one_row(q_row, k0, v0, (int64_t)c->Hkv * c->D, n, n - 1, c->D, c->scale,
                   c->o + r * c->D, c->lse + r, scratch);
}

static int check_decode(const int32_t* seqlens, int B, int Hq, int Hkv, int D, int Lmax) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0 || Hq % Hkv) return 1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 1 || seqlens[b] > Lmax) return 1;
    return 0;
}

int oracle_decode_rows(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                       const int32_t* seqlens, int B, int Hq, int Hkv, int D, int Lmax,
                       double scale, const int64_t* rows, int64_t nrows,
                       double* o, double* lse, int nthreads) {
    if (check_decode(seqlens, B, Hq, Hkv, D, Lmax)) return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq) return 2;
    dec_ctx c = {q, k_cache, v_cache, seqlens, B, Hq, Hkv, D, Lmax, 0, scale, rows, o, lse};
    return parallel_rows(decode_row_task, &c, nrows, (size_t)Lmax, nthreads);
}

/* Chunking of a sequence of n keys into S splits: chunk size
 * C = 64 * ceil(ceil(n / S) / 64); chunk c covers [c*C, min((c+1)*C, n)),
 * possibly empty.  The chunk boundaries do not change the exact result. */
static void decode_split_row_task(void* vctx, int64_t r, double* scratch) {
    const dec_ctx* c = (const dec_ctx*)vctx;
    int64_t flat = c->rows[r];
    int h = (int)(flat % c->Hq), b = (int)(flat / c->Hq);
    int g = h / (c->Hq / c->Hkv);
    int D = c->D, S = c->S;
    int64_t n = c->seqlens[b];
    int64_t per = (n + S - 1) / S;
    int64_t C = ((per + 63) / 64) * 64;
    double* o_parts = scratch;                 /* S * D */
    double* l_parts = scratch + (int64_t)S * D; /* S */
    double* s = l_parts + S;                   /* Lmax */
    const uint16_t* q_row = c->q + ((int64_t)b * c->Hq + h) * D;
    int64_t stride = (int64_t)c->Hkv * D;
    for (int ci = 0; ci < S; ++ci) {
        int64_t j0 = (int64_t)ci * C, j1 = j0 + C < n ? j0 + C : n;
        if (j0 >= j1) {
            l_parts[ci] = -INFINITY;
            for (int d = 0; d < D; ++d) o_parts[(int64_t)ci * D + d] = 0.0;
            continue;
        }
        const uint16_t* k0 = c->kc + (((int64_t)b * c->Lmax + j0) * c->Hkv + g) * D;
        const uint16_t* v0 = c->vc + (((int64_t)b * c->Lmax + j0) * c->Hkv + g) * D;
        attend_one_row(q_row, k0, v0, stride, j1 - j0, j1 - j0 - 1, D, c->scale,
                       o_parts + (int64_t)ci * D, &l_parts[ci], s);
    }
    oracle_lse_merge(o_parts, l_parts, S, D, c->o + r * D, c->lse + r);
}

int oracle_decode_split_rows(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                             const int32_t* seqlens, int B, int Hq, int Hkv, int D, int Lmax,
                             int num_splits, double scale, const int64_t* rows, int64_t nrows,
                             double* o, double* lse, int nthreads) {
    if (check_decode(seqlens, B, Hq, Hkv, D, Lmax) || num_splits < 1) return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq) return 2;
    dec_ctx c = {q, k_cache, v_cache, seqlens, B, Hq, Hkv, D, Lmax, num_splits, scale, rows, o, lse};
    size_t scratch = (size_t)num_splits * D + (size_t)num_splits + (size_t)Lmax;
    return parallel_rows(decode_split_row_task, &c, nrows, scratch, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Decode against a paged cache.                                             */
/* pool [num_pages, page_size, Hkv, D]; table [B, max_pages]; rows b*Hq + h. */
/* ------------------------------------------------------------------------- */
typedef struct {
    const uint16_t *q, *kp, *vp;
    const int32_t *table, *seqlens;
    int B, Hq, Hkv, D, num_pages, page_size, max_pages;
    double scale;
    const int64_t* rows;
    double *o, *lse;
} paged_ctx;

/* Address of key j of sequence b, kv head g, in a pool. */
static const uint16_t* paged_row(const paged_ctx* c, const uint16_t* pool, int b, int64_t j, int g) {
    int64_t page = c->table[(int64_t)b * c->max_pages + j / c->page_size];
    int64_t row = j % c->page_size;
    return pool + ((page * c->page_size + row) * c->Hkv + g) * c->D;
}

static void paged_row_task(void* vctx, int64_t r, double* s) {
    const paged_ctx* c = (const paged_ctx*)vctx;
    int64_t flat = c->rows[r];
    int h = (int)(flat % c->Hq), b = (int)(flat / c->Hq);
    int g = h / (c->Hq / c->Hkv);
    int D = c->D;
    int64_t n = c->seqlens[b];
    const uint16_t* q_row = c->q + ((int64_t)b * c->Hq + h) * D;
    double* o = c->o + r * D;
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        const uint16_t* kr = paged_row(c, c->kp, b, j, g);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(kr[d]);
        s[j] = c->scale * dot;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double p = exp(s[j] - m);
        sum += p;
        const uint16_t* vr = paged_row(c, c->vp, b, j, g);
        for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_double(vr[d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= sum;
    c->lse[r] = m + log(sum);
}

int oracle_decode_paged_rows(const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                             const int32_t* block_table, const int32_t* seqlens, int B, int Hq, int Hkv,
                             int D, int num_pages, int page_size, int max_pages, double scale,
                             const int64_t* rows, int64_t nrows, double* o, double* lse, int nthreads) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv || num_pages <= 0 || page_size <= 0 ||
        max_pages <= 0)
        return 1;
    for (int b = 0; b < B; ++b) {
        int64_t n = seqlens[b];
        if (n < 1 || n > (int64_t)max_pages * page_size) return 1;
        for (int64_t lp = 0; lp < (n + page_size - 1) / page_size; ++lp) {
            int32_t pg = block_table[(int64_t)b * max_pages + lp];
            if (pg < 0 || pg >= num_pages) return 3;
        }
    }
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq) return 2;
    paged_ctx c = {q, k_pages, v_pages, block_table, seqlens, B, Hq, Hkv, D, num_pages, page_size, max_pages,
                   scale, rows, o, lse};
    return parallel_rows(paged_row_task, &c, nrows, (size_t)max_pages * page_size, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Packed variable-length batch: q [total_q, Hq, D], k/v [total_k, Hkv, D];   */
/* sequence b holds query tokens [cu_q[b], cu_q[b+1]) and keys                */
/* [cu_k[b], cu_k[b+1]).  rows: flat t*Hq + h over packed query tokens t.     */
/* ------------------------------------------------------------------------- */
typedef struct {
    const uint16_t *q, *k, *v;
    const int32_t *cu_q, *cu_k;
    int B, total_q, total_k, Hq, Hkv, D, causal;
    double scale;
    const int64_t* rows;
    double *o, *lse;
} varlen_ctx;

static void varlen_row_task(void* vctx, int64_t r, double* scratch) {
    const varlen_ctx* c = (const varlen_ctx*)vctx;
    int64_t flat = c->rows[r];
    int64_t t = flat / c->Hq;
    int h = (int)(flat % c->Hq);
    int b = 0;
    while (b + 1 < c->B && c->cu_q[b + 1] <= t) ++b;   /* sequence holding token t */
    int64_t i = t - c->cu_q[b];
    int64_t Lq = c->cu_q[b + 1] - c->cu_q[b], Lk = c->cu_k[b + 1] - c->cu_k[b];
    int64_t limit = c->causal ? i + (Lk - Lq) : Lk - 1;
    double* o = c->o + r * c->D;
    if (Lk == 0 || limit < 0) {                       /* no allowed key */
        for (int d = 0; d < c->D; ++d) o[d] = 0.0;
        c->lse[r] = -INFINITY;
        return;
    }
    int g = h / (c->Hq / c->Hkv);
    const uint16_t* q_row = c->q + (t * c->Hq + h) * c->D;
    const uint16_t* k0 = c->k + ((int64_t)c->cu_k[b] * c->Hkv + g) * c->D;
    const uint16_t* v0 = c->v + ((int64_t)c->cu_k[b] * c->Hkv + g) * c->D;
    attend_one_row(q_row, k0, v0, (int64_t)c->Hkv * c->D, Lk, limit, c->D, c->scale, o, c->lse + r, scratch);
}

int oracle_attention_varlen_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const int32_t* cu_q, const int32_t* cu_k, int B, int total_q, int total_k,
                                 int Hq, int Hkv, int D, double scale, int causal,
                                 const int64_t* rows, int64_t nrows, double* o, double* lse, int nthreads) {
    if (B <= 0 || total_q <= 0 || total_k < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv) return 1;
    if (cu_q[0] != 0 || cu_k[0] != 0 || cu_q[B] != total_q || cu_k[B] != total_k) return 1;
    int64_t max_lk = 0;
    for (int b = 0; b < B; ++b) {
        if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b]) return 1;
        if (cu_k[b + 1] - cu_k[b] > max_lk) max_lk = cu_k[b + 1] - cu_k[b];
    }
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)total_q * Hq) return 2;
    varlen_ctx c = {q, k, v, cu_q, cu_k, B, total_q, total_k, Hq, Hkv, D, causal, scale, rows, o, lse};
    return parallel_rows(varlen_row_task, &c, nrows, (size_t)(max_lk > 0 ? max_lk : 1), nthreads);
}

/* ------------------------------------------------------------------------- */
/* KV-INT8.  The pages name int8 K (and V) caches but not the granularity;    */
/* the reading used here: symmetric, one scale per (b, token, kv head)        */
/* vector of D values, scale = max|x| / 127, code = round-half-even(x/scale)  */
/* clamped to [-127, 127]; an all-zero vector gets scale 0 and codes 0.       */
/* The steps are fp32 (the precision the kernels decide the codes in):        */
/* fp32 division correctly rounded, rintf in the default rounding mode.      */
/* x: [B, L, H, D] bf16; codes: [B, L, H, D] int8; scales: [B, H, L] fp32.    */
/* ------------------------------------------------------------------------- */
int oracle_quantize_kv_int8(const uint16_t* x, int8_t* codes, float* scales, int B, int L, int H, int D) {
    if (B <= 0 || L <= 0 || H <= 0 || D <= 0) return 1;
    if (fegetround() != FE_TONEAREST) return 2;
    for (int b = 0; b < B; ++b)
        for (int j = 0; j < L; ++j)
            for (int h = 0; h < H; ++h) {
                const uint16_t* xr = x + (((int64_t)b * L + j) * H + h) * D;
                int8_t* cr = codes + (((int64_t)b * L + j) * H + h) * D;
                float amax = 0.0f;
                for (int d = 0; d < D; ++d) {
                    float a = fabsf((float)bf16_bits_to_double(xr[d]));
                    if (a > amax) amax = a;
                }
                float sc = amax / 127.0f;
                scales[((int64_t)b * H + h) * L + j] = sc;
                for (int d = 0; d < D; ++d) {
                    if (amax == 0.0f) { cr[d] = 0; continue; }
                    float r = rintf((float)bf16_bits_to_double(xr[d]) / sc);
                    if (r > 127.0f) r = 127.0f;
                    if (r < -127.0f) r = -127.0f;
                    cr[d] = (int8_t)r;
                }
            }
    return 0;
}

/* Decode against an int8 cache: k codes [B, Lmax, Hkv, D] int8 with k scales */
/* [B, Hkv, Lmax]; v either int8 codes + scales (v_int8 = 1) or bf16.         */
typedef struct {
    const uint16_t* q;
    const int8_t* kc;
    const float* ks;
    const void* vc;
    const float* vs;
    int v_int8;
    const int32_t* seqlens;
    int B, Hq, Hkv, D, Lmax;
    double scale;
    const int64_t* rows;
    double *o, *lse;
} dec8_ctx;

static void decode_int8_row_task(void* vctx, int64_t r, double* s) {
    const dec8_ctx* c = (const dec8_ctx*)vctx;
    int64_t flat = c->rows[r];
    int h = (int)(flat % c->Hq), b = (int)(flat / c->Hq);
    int g = h / (c->Hq / c->Hkv);
    int D = c->D;
    int64_t n = c->seqlens[b];
    const uint16_t* q_row = c->q + ((int64_t)b * c->Hq + h) * D;
    double* o = c->o + r * D;
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        const int8_t* kr = c->kc + (((int64_t)b * c->Lmax + j) * c->Hkv + g) * D;
        double ksc = (double)c->ks[((int64_t)b * c->Hkv + g) * c->Lmax + j];
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_bits_to_double(q_row[d]) * (ksc * (double)kr[d]);
        s[j] = c->scale * dot;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double p = exp(s[j] - m);
        sum += p;
        int64_t vrow = (((int64_t)b * c->Lmax + j) * c->Hkv + g) * D;
        if (c->v_int8) {
            const int8_t* vr = (const int8_t*)c->vc + vrow;
            double vsc = (double)c->vs[((int64_t)b * c->Hkv + g) * c->Lmax + j];
            for (int d = 0; d < D; ++d) o[d] += p * (vsc * (double)vr[d]);
        } else {
            const uint16_t* vr = (const uint16_t*)c->vc + vrow;
            for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_double(vr[d]);
        }
    }
    for (int d = 0; d < D; ++d) o[d] /= sum;
    c->lse[r] = m + log(sum);
}

int oracle_decode_int8_rows(const uint16_t* q, const int8_t* k_codes, const float* k_scales,
                            const void* v_cache, const float* v_scales, int v_int8,
                            const int32_t* seqlens, int B, int Hq, int Hkv, int D, int Lmax, double scale,
                            const int64_t* rows, int64_t nrows, double* o, double* lse, int nthreads) {
    if (check_decode(seqlens, B, Hq, Hkv, D, Lmax)) return 1;
    if (v_int8 && !v_scales) return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq) return 2;
    dec8_ctx c = {q, k_codes, k_scales, v_cache, v_scales, v_int8, seqlens, B, Hq, Hkv, D, Lmax, scale, rows, o, lse};
    return parallel_rows(decode_int8_row_task, &c, nrows, (size_t)Lmax, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Backward: for loss-gradient dO [B, Lq, Hq, D] (bf16), the gradients of     */
/* the definition w.r.t. q, k, v, in fp64 (dq [B,Lq,Hq,D], dk/dv             */
/* [B,Lk,Hkv,D]).  One (b, h_q) problem at a time: the full P and dP rows.    */
/* The chain rule through softmax: with O = P V, dV = P^T dO; dP = dO V^T;    */
/* dS_ij = P_ij (dP_ij - sum_l P_il dP_il), and sum_l P_il dP_il =            */
/* sum_d dO_id O_id; scores s = scale q.k, so dQ = scale dS K and             */
/* dK = scale dS^T Q.  Masked entries have P = 0 and contribute nothing.      */
/* ------------------------------------------------------------------------- */
int oracle_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                              int B, int Lq, int Lk, int Hq, int Hkv, int D, double scale, int causal,
                              double* dq, double* dk, double* dv) {
    if (check_shape(B, Lq, Lk, Hq, Hkv, D, causal)) return 1;
    const int G = Hq / Hkv;
    double* P = (double*)malloc((size_t)Lq * Lk * sizeof(double));
    double* dP = (double*)malloc((size_t)Lq * Lk * sizeof(double));
    double* O = (double*)malloc((size_t)Lq * D * sizeof(double));
    if (!P || !dP || !O) { free(P); free(dP); free(O); return 4; }
    memset(dq, 0, (size_t)B * Lq * Hq * D * sizeof(double));
    memset(dk, 0, (size_t)B * Lk * Hkv * D * sizeof(double));
    memset(dv, 0, (size_t)B * Lk * Hkv * D * sizeof(double));
#define QX(b, i, h, d) bf16_bits_to_double(q[(((int64_t)(b) * Lq + (i)) * Hq + (h)) * D + (d)])
#define DOX(b, i, h, d) bf16_bits_to_double(dout[(((int64_t)(b) * Lq + (i)) * Hq + (h)) * D + (d)])
#define KX(b, j, g, d) bf16_bits_to_double(k[(((int64_t)(b) * Lk + (j)) * Hkv + (g)) * D + (d)])
#define VX(b, j, g, d) bf16_bits_to_double(v[(((int64_t)(b) * Lk + (j)) * Hkv + (g)) * D + (d)])
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            for (int i = 0; i < Lq; ++i) {          /* P row i: the definition */
                int64_t limit = causal ? i + (int64_t)(Lk - Lq) : (int64_t)Lk - 1;
                double m = -INFINITY;
                for (int j = 0; j < Lk; ++j) {
                    double sc = -INFINITY;
                    if (j <= limit) {
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d) dot += QX(b, i, h, d) * KX(b, j, g, d);
                        sc = scale * dot;
                    }
                    P[(int64_t)i * Lk + j] = sc;
                    if (sc > m) m = sc;
                }
                double z = 0.0;
                for (int j = 0; j < Lk; ++j) {
                    double e = (P[(int64_t)i * Lk + j] == -INFINITY) ? 0.0 : exp(P[(int64_t)i * Lk + j] - m);
                    P[(int64_t)i * Lk + j] = e;
                    z += e;
                }
                for (int j = 0; j < Lk; ++j) P[(int64_t)i * Lk + j] /= z;
                for (int d = 0; d < D; ++d) {      /* O = P V */
                    double acc = 0.0;
                    for (int j = 0; j < Lk; ++j) acc += P[(int64_t)i * Lk + j] * VX(b, j, g, d);
                    O[(int64_t)i * D + d] = acc;
                }
                for (int j = 0; j < Lk; ++j) {      /* dP = dO V^T */
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += DOX(b, i, h, d) * VX(b, j, g, d);
                    dP[(int64_t)i * Lk + j] = acc;
                }
            }
            for (int i = 0; i < Lq; ++i) {
                double delta = 0.0;                 /* rowsum(dO o O) */
                for (int d = 0; d < D; ++d) delta += DOX(b, i, h, d) * O[(int64_t)i * D + d];
                for (int j = 0; j < Lk; ++j) {
                    double pij = P[(int64_t)i * Lk + j];
                    if (pij == 0.0) continue;
                    double ds = pij * (dP[(int64_t)i * Lk + j] - delta);
                    double* dqr = dq + (((int64_t)b * Lq + i) * Hq + h) * D;
                    double* dkr = dk + (((int64_t)b * Lk + j) * Hkv + g) * D;
                    double* dvr = dv + (((int64_t)b * Lk + j) * Hkv + g) * D;
                    for (int d = 0; d < D; ++d) {
                        dqr[d] += scale * ds * KX(b, j, g, d);
                        dkr[d] += scale * ds * QX(b, i, h, d);
                        dvr[d] += pij * DOX(b, i, h, d);
                    }
                }
            }
        }
#undef QX
#undef DOX
#undef KX
#undef VX
    free(P);
    free(dP);
    free(O);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* e4m3 (OCP 8-bit float, E4M3 variant).                                     */
/* ------------------------------------------------------------------------- */
static double e4m3_value(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m, -9)              /* subnormal: m * 2^-9 */
                              : ldexp(1.0 + m / 8.0, e - 7);       /* normal: 1.m * 2^(e-7) */
    return sign ? -mag : mag;
}

/* Round to nearest (ties to even), saturating finite values at +-448. */
static uint8_t e4m3_code(float x) {
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return sign | 0x7F;
    const double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {                       /* subnormal range: multiples of 2^-9 */
        const int m = (int)nearbyint(a * 512.0);    /* 8 lands on the smallest normal, code 0x08 */
        return sign | (uint8_t)m;
    }
    int ex;
    const double f = frexp(a, &ex);                 /* a = f 2^ex, f in [1/2, 1) */
    int e = ex - 1;                                 /* a = (2f) 2^e, 2f in [1, 2) */
    int m = (int)nearbyint((2.0 * f - 1.0) * 8.0);  /* exact product; ties to even */
    if (m == 8) { m = 0; ++e; }
    if (e > 8 || (e == 8 && m == 7)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | m);
}

int oracle_e4m3_decode(const uint8_t* c, int64_t n, double* out) {
    if (n < 0) return 1;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(c[i]);
    return 0;
}

int oracle_e4m3_encode(const float* x, int64_t n, uint8_t* out) {
    if (n < 0) return 1;
    if (fegetround() != FE_TONEAREST) return 2;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_code(x[i]);
    return 0;
}

/* x [B, L, H, D] bf16 bits -> codes [B, L, H, D], descale [B, H]. */
int oracle_quantize_fp8(const uint16_t* x, uint8_t* codes, float* descale, int B, int L, int H, int D) {
    if (B <= 0 || L <= 0 || H <= 0 || D <= 0) return 1;
    if (fegetround() != FE_TONEAREST) return 2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            float amax = 0.0f;
            for (int j = 0; j < L; ++j)
                for (int d = 0; d < D; ++d) {
                    const float a = fabsf((float)bf16_bits_to_double(x[(((int64_t)b * L + j) * H + h) * D + d]));
                    if (a > amax) amax = a;
                }
            /* amax below 2^-110 (zero, or small enough for 448 / amax to leave
               the fp32 range): inv = descale = 1 */
            const int tiny = amax < ldexpf(1.0f, -110);
            const float inv = tiny ? 1.0f : 448.0f / amax;
            descale[(int64_t)b * H + h] = tiny ? 1.0f : amax / 448.0f;
            for (int j = 0; j < L; ++j)
                for (int d = 0; d < D; ++d) {
                    const int64_t e = (((int64_t)b * L + j) * H + h) * D + d;
                    const float y = (float)bf16_bits_to_double(x[e]) * inv;
                    codes[e] = e4m3_code(y);
                }
        }
    return 0;
}

typedef struct {
    const uint8_t *q, *k, *v;
    const float *qd, *kd, *vd;
    int B, Lq, Lk, Hq, Hkv, D, causal;
    double scale;
    const int64_t* rows;
    double *o, *lse;
} fp8_ctx;

static void fp8_row_task(void* vctx, int64_t r, double* s) {
    const fp8_ctx* c = (const fp8_ctx*)vctx;
    const int64_t flat = c->rows[r];
    const int64_t i = flat % c->Lq;
    const int h = (int)((flat / c->Lq) % c->Hq);
    const int b = (int)(flat / ((int64_t)c->Lq * c->Hq));
    const int g = h / (c->Hq / c->Hkv);
    const int D = c->D;
    const double qs = c->qd[(int64_t)b * c->Hq + h];
    const double ks = c->kd[(int64_t)b * c->Hkv + g];
    const double vs = c->vd[(int64_t)b * c->Hkv + g];
    const uint8_t* q_row = c->q + (((int64_t)b * c->Lq + i) * c->Hq + h) * D;
    const int64_t limit = c->causal ? i + (int64_t)(c->Lk - c->Lq) : (int64_t)c->Lk - 1;
    double m = -INFINITY;
    for (int64_t j = 0; j < c->Lk; ++j) {
        if (j > limit) { s[j] = -INFINITY; continue; }
        const uint8_t* kr = c->k + (((int64_t)b * c->Lk + j) * c->Hkv + g) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += (e4m3_value(q_row[d]) * qs) * (e4m3_value(kr[d]) * ks);
        s[j] = c->scale * dot;
        if (s[j] > m) m = s[j];
    }
    double* o = c->o + r * D;
    double sum = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < c->Lk; ++j) {
        if (s[j] == -INFINITY) continue;
        const double p = exp(s[j] - m);
        sum += p;
        const uint8_t* vr = c->v + (((int64_t)b * c->Lk + j) * c->Hkv + g) * D;
        for (int d = 0; d < D; ++d) o[d] += p * (e4m3_value(vr[d]) * vs);
    }
    for (int d = 0; d < D; ++d) o[d] /= sum;
    c->lse[r] = m + log(sum);
}

/* q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D] e4m3 codes; qd [B,Hq], kd/vd [B,Hkv];
 * rows: flat (b*Hq+h)*Lq+i; o [nrows, D], lse [nrows]. */
int oracle_attention_fp8_rows(const uint8_t* q, const uint8_t* k, const uint8_t* v, const float* qd,
                              const float* kd, const float* vd, int B, int Lq, int Lk, int Hq, int Hkv, int D,
                              double scale, int causal, const int64_t* rows, int64_t nrows, double* o,
                              double* lse, int nthreads) {
    if (check_shape(B, Lq, Lk, Hq, Hkv, D, causal)) return 1;
    const int64_t total = (int64_t)B * Hq * Lq;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return 2;
    fp8_ctx c = {q, k, v, qd, kd, vd, B, Lq, Lk, Hq, Hkv, D, causal, scale, rows, o, lse};
    return parallel_rows(fp8_row_task, &c, nrows, (size_t)Lk, nthreads);
}
