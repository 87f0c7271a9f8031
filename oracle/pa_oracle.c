/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for paged-KV attention.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load this library. The product (the CUDA
 * library and its Python binding) never calls, links or imports it, and it
 * shares no code, header or table with the CUDA kernels.
 *
 * What each function follows (cited by page title and section):
 *
 *  [KV]  page "字节跳动 AI Infra (2)", question "KV Cache原理与优化" (KV cache
 *        principle), the per-step formulas: the new token's K_t/V_t are
 *        appended to the cache, K_cache = concat(K_cache, K_t), and the step's
 *        output is softmax(Q_t . K_cache^T / sqrt(d)) . V_cache, shape [1, d].
 *  [PG]  same page, question "vLLM与PagedAttention的原理" (PagedAttention
 *        principle): a pool of fixed-size physical blocks (16 tokens of K/V
 *        each in the example), a per-request block table mapping logical block
 *        i to a physical block id, and the kernel sketch that finds a block's
 *        keys at k_cache + physical_block * block_size * head_dim.
 *  [GQA] page "LLM推理优化", section 1.3 (KV cache optimisation strategies):
 *        under GQA several query heads share one K/V head; under MQA all do.
 *  [FD]  page "字节跳动 AI Infra (2)", question "推理加速的综合策略有哪些",
 *        table of algorithm-level optimisations, row FlashDecoding: decode is
 *        parallelised by splitting along the KV length.
 *  [Q8]  page "字节跳动 AI Infra (2)", optimisation table, row "KV量化(INT8)"
 *        (store K/V in low precision, halving the cache), and page
 *        "LLM推理优化", section 1.3 (quantise K/V from FP16 to INT8/INT4):
 *        here INT8 codes or FP8 E4M3 codes, one scale per K/V head,
 *        value = code * scale.
 *  [SW]  page "LLM推理优化", section 2.3 (flash_attn_func window_size) and page
 *        "vLLM框架是怎么做推理加速的", 追问 3 (sliding window attention): a query
 *        sees only the last `window` positions up to its own.
 *  [CP]  page "vLLM框架是怎么做推理加速的", section 3 (Chunked Prefill): a
 *        prompt is cut into chunks (512 tokens by default) that attend over
 *        the cache; page "LLM推理优化", section 2.3: prefill attention is
 *        causal (flash_attn_func(..., causal=True)).
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes):
 *  - Cache layout [num_blocks][num_kv_heads][block_size][head_dim]; the page's
 *    pointer formula is the num_kv_heads == 1 case of it.
 *  - Query head h reads K/V head h / (H_q / H_kv) (contiguous groups).
 *  - The scale is a parameter (the pages use 1/sqrt(d)).
 *  - context_lens[b] counts the valid tokens of sequence b, including the one
 *    just appended; table entries and slots past it are never read.
 *  - A sequence with no tokens yields out = 0 and lse = -inf.
 *  - Chunk queries are bottom-right aligned: query i of a chunk of C queries
 *    over ctx tokens sits at position ctx - C + i and attends keys 0..that
 *    position. The chunk's own K/V are already in the cache.
 *  - Stored values (fp32, or bf16 bit patterns) are widened exactly to double;
 *    everything after that is plain fp64 arithmetic.
 *  - softmax is evaluated as exp(s - max s) / sum exp(s - max s), which is the
 *    definition multiplied through by exp(-max s) / exp(-max s).
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fPIC -shared.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2, OR_I8 = 3 };
enum { OR_OK = 0, OR_BAD_SLOT = 1, OR_BAD_BLOCK = 2, OR_BAD_ARG = 3, OR_NO_MEM = 4 };

/* [Q8] value of an FP8 E4M3 code (1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9; no
 * infinities; S.1111.111 is NaN; largest finite magnitude 448). */
static double e4m3_value(uint8_t c)
{
    int e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if ((c & 0x7F) == 0x7F) return NAN;
    if (e == 0)
        v = m * ldexp(1.0, -9);
    else
        v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* [Q8] code of the E4M3 value nearest to x, ties to the even code, finite
 * magnitudes beyond 448 (and infinities) saturated to +-448, NaN to 0x7F.
 * Written as a plain search over the 127 non-negative codes. */
uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    int k = 0; /* largest code with value <= a */
    while (k + 1 <= 0x7E && e4m3_value((uint8_t)(k + 1)) <= a) ++k;
    double lo = e4m3_value((uint8_t)k), hi = e4m3_value((uint8_t)(k + 1));
    int code;
    if (a - lo < hi - a)
        code = k;
    else if (a - lo > hi - a)
        code = k + 1;
    else
        code = (k % 2 == 0) ? k : k + 1;
    return sign | (uint8_t)code;
}

double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }

/* [Q8] INT8 code of q, an fp32 quotient x / scale: the nearest integer, ties
 * to even (the default rounding mode of nearbyint), saturated to the
 * symmetric range [-127, 127]; NaN gives 0. */
int8_t oracle_int8_encode(float q)
{
    if (isnan(q)) return 0;
    double r = nearbyint((double)q);
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int8_t)r;
}

/* A stored element, widened exactly to double. bf16 is the top half of an
 * IEEE binary32, so shifting its 16 bits up gives the same number as a float.
 * An E4M3 or INT8 code is its value times the K/V head's scale (exact in
 * double). */
static double stored_scaled(const void *base, int64_t i, int dtype, double scale)
{
    if (dtype == OR_F32) return (double)((const float *)base)[i];
    if (dtype == OR_E4M3) return e4m3_value(((const uint8_t *)base)[i]) * scale;
    if (dtype == OR_I8) return (double)((const int8_t *)base)[i] * scale;
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double stored(const void *base, int64_t i, int dtype)
{
    return stored_scaled(base, i, dtype, 1.0);
}

/* One sequence's view of the pool: where its block table row is and which
 * K/V head is being read. */
typedef struct {
    const void *k_cache, *v_cache;
    int dtype;
    const int32_t *table_row; /* block_tables[b][0 .. max_blocks_per_seq) */
    int max_blocks;
    int H_kv, D, bs;
    int64_t NB;
    int kv_head;
    double k_scale, v_scale; /* 8-bit caches: value = code * scale */
} paged_seq;

/* [PG] element index of K/V[position j][dim 0] of this sequence and head:
 * logical block j / bs is looked up in the table; the token sits at offset
 * j % bs inside the physical block. Returns -1 for an id outside the pool. */
static int64_t token_base(const paged_seq *s, int64_t j)
{
    int64_t logical_block = j / s->bs;
    int64_t offset = j % s->bs;
    if (logical_block >= s->max_blocks) return -1;
    int64_t phys = s->table_row[logical_block];
    if (phys < 0 || phys >= s->NB) return -1;
    return ((phys * s->H_kv + s->kv_head) * s->bs + offset) * s->D;
}

/* [KV] one query vector q[0..D) against the sequence's keys at positions
 * [j0, j1): scores s_j = scale * (q . K_j), weights softmax(s), output
 * sum_j softmax(s)_j V_j, and lse = log sum_j exp(s_j).
 * sbuf must hold j1 - j0 doubles. */
static int attend(double *o, double *lse, const double *q, const paged_seq *s,
                  int64_t j0, int64_t j1, double scale, double *sbuf)
{
    const int D = s->D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (j1 <= j0) {
        *lse = -INFINITY;
        return OR_OK;
    }
    double m = -INFINITY;
    for (int64_t j = j0; j < j1; ++j) {
        int64_t base = token_base(s, j);
        if (base < 0) return OR_BAD_BLOCK;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += q[d] * stored_scaled(s->k_cache, base + d, s->dtype, s->k_scale);
        double sc = scale * dot;
        sbuf[j - j0] = sc;
        if (sc > m) m = sc;
    }
    double denom = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
        double p = exp(sbuf[j - j0] - m);
        sbuf[j - j0] = p;
        denom += p;
    }
    for (int64_t j = j0; j < j1; ++j) {
        int64_t base = token_base(s, j);
        double w = sbuf[j - j0] / denom;
        for (int d = 0; d < D; ++d)
            o[d] += w * stored_scaled(s->v_cache, base + d, s->dtype, s->v_scale);
    }
    *lse = m + log(denom);
    return OR_OK;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* [KV]+[PG] the append step in paged form. For each new token t with slot
 * s = slot_mapping[t] >= 0, the token's K/V rows for every K/V head are copied
 * into physical block s / bs at offset s % bs. Negative slots are padding and
 * are skipped. A slot past the pool returns OR_BAD_SLOT before anything is
 * written. Element type does not matter: the copy is of bytes. */
int oracle_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                             const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int64_t num_blocks, int elem_bytes)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || elem_bytes <= 0)
        return OR_BAD_ARG;
    for (int64_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_blocks * (int64_t)block_size) return OR_BAD_SLOT;
    const size_t row = (size_t)head_dim * (size_t)elem_bytes;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / block_size, offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t src = ((size_t)t * num_kv_heads + h) * row;
            size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * row;
            memcpy((char *)k_cache + dst, (const char *)key + src, row);
            memcpy((char *)v_cache + dst, (const char *)value + src, row);
        }
    }
    return OR_OK;
}

/* Shared argument checks for the attention entry points. */
static int check_heads(int H_q, int H_kv, int D, int bs, int MB, int64_t NB)
{
    if (H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0 || D <= 0 || bs <= 0 || MB < 0 || NB <= 0)
        return OR_BAD_ARG;
    return OR_OK;
}

/* [KV]+[PG]+[GQA] decode: for every sequence b and query head h (or only the
 * pairs with select[b*H_q+h] != 0), attend q[b][h] over positions
 * [0, context_lens[b]) gathered through block_tables[b], reading K/V head
 * h / (H_q/H_kv). out: [B][H_q][D] doubles; lse: [B][H_q] (may be NULL). */
int oracle_decode(double *out, double *lse, const void *q, const void *k_cache,
                  const void *v_cache, int dtype, const int32_t *block_tables,
                  const int32_t *context_lens, int B, int H_q, int H_kv, int D, int bs, int MB,
                  int64_t NB, double scale, const uint8_t *select)
{
    int rc = check_heads(H_q, H_kv, D, bs, MB, NB);
    if (rc) return rc;
    for (int b = 0; b < B; ++b)
        if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs) return OR_BAD_ARG;
    const int group = H_q / H_kv;
    int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : err)
    for (int64_t bh = 0; bh < (int64_t)B * H_q; ++bh) {
        if (select && !select[bh]) continue;
        int b = (int)(bh / H_q), h = (int)(bh % H_q);
        paged_seq s = {k_cache, v_cache, dtype, block_tables + (int64_t)b * MB, MB,
                       H_kv, D, bs, NB, h / group, 1.0, 1.0};
        double *qv = malloc(sizeof(double) * D);
        double *sbuf = malloc(sizeof(double) * (context_lens[b] > 0 ? context_lens[b] : 1));
        if (!qv || !sbuf) {
            free(qv); free(sbuf);
            err = OR_NO_MEM > err ? OR_NO_MEM : err;
            continue;
        }
        for (int d = 0; d < D; ++d) qv[d] = stored(q, bh * D + d, dtype);
        double l;
        int r = attend(out + bh * D, &l, qv, &s, 0, context_lens[b], scale, sbuf);
        if (lse) lse[bh] = l;
        if (r > err) err = r;
        free(qv);
        free(sbuf);
    }
    return err;
}

/* [FD] the same decode restricted to KV partitions: partition p of sequence b
 * covers positions [p*partition_tokens, min((p+1)*partition_tokens, ctx_b)).
 * o_parts: [B][H_q][S][D], lse_parts: [B][H_q][S]; partitions past the end of
 * a sequence hold o = 0, lse = -inf. */
int oracle_decode_partials(double *o_parts, double *lse_parts, const void *q, const void *k_cache,
                           const void *v_cache, int dtype, const int32_t *block_tables,
                           const int32_t *context_lens, int B, int H_q, int H_kv, int D, int bs,
                           int MB, int64_t NB, double scale, int partition_tokens, int S)
{
    int rc = check_heads(H_q, H_kv, D, bs, MB, NB);
    if (rc) return rc;
    if (partition_tokens <= 0 || S <= 0) return OR_BAD_ARG;
    for (int b = 0; b < B; ++b)
        if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs ||
            (int64_t)context_lens[b] > (int64_t)S * partition_tokens)
            return OR_BAD_ARG;
    const int group = H_q / H_kv;
    int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : err)
    for (int64_t bh = 0; bh < (int64_t)B * H_q; ++bh) {
        int b = (int)(bh / H_q), h = (int)(bh % H_q);
        paged_seq s = {k_cache, v_cache, dtype, block_tables + (int64_t)b * MB, MB,
                       H_kv, D, bs, NB, h / group, 1.0, 1.0};
        double *qv = malloc(sizeof(double) * D);
        double *sbuf = malloc(sizeof(double) * partition_tokens);
        if (!qv || !sbuf) {
            free(qv); free(sbuf);
            err = OR_NO_MEM > err ? OR_NO_MEM : err;
            continue;
        }
        for (int d = 0; d < D; ++d) qv[d] = stored(q, bh * D + d, dtype);
        for (int p = 0; p < S; ++p) {
            int64_t j0 = (int64_t)p * partition_tokens;
            int64_t j1 = j0 + partition_tokens;
            if (j1 > context_lens[b]) j1 = context_lens[b];
            int r = attend(o_parts + (bh * S + p) * D, lse_parts + bh * S + p, qv, &s, j0, j1,
                           scale, sbuf);
            if (r > err) err = r;
        }
        free(qv);
        free(sbuf);
    }
    return err;
}

/* [FD] merge of partial results by log-sum-exp. With L = log sum_s exp(lse_s),
 * out = sum_s exp(lse_s - L) o_s, which equals attention over the union of the
 * partitions because each o_s is already normalised by its own exp(lse_s).
 * Partitions with lse = -inf carry no weight; if all do, out = 0, lse = -inf.
 * o_parts: [R][S][D], lse_parts: [R][S], out: [R][D], lse: [R]. */
void oracle_lse_merge(double *out, double *lse, const double *o_parts, const double *lse_parts,
                      int64_t R, int S, int D)
{
    for (int64_t r = 0; r < R; ++r) {
        const double *ls = lse_parts + r * S;
        double m = -INFINITY;
        for (int p = 0; p < S; ++p)
            if (ls[p] > m) m = ls[p];
        for (int d = 0; d < D; ++d) out[r * D + d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double total = 0.0;
        for (int p = 0; p < S; ++p) total += exp(ls[p] - m);
        for (int p = 0; p < S; ++p) {
            if (ls[p] == -INFINITY) continue;
            double w = exp(ls[p] - m) / total;
            for (int d = 0; d < D; ++d) out[r * D + d] += w * o_parts[(r * S + p) * D + d];
        }
        lse[r] = m + log(total);
    }
}

/* [CP] chunked prefill. Chunk c owns query rows [qsl[c], qsl[c+1]) of q
 * ([total_q][H_q][D]) and block_tables[c]; context_lens[c] is its total
 * context (cached tokens plus the chunk's own C tokens, all in the cache).
 * Query i attends positions [0, ctx - C + i] (causal, bottom-right aligned).
 * out: [total_q][H_q][D]; lse: [total_q][H_q] (may be NULL); select as in
 * oracle_decode over (row, head). */
static int prefill_impl(double *out, double *lse, const void *q, const void *k_cache,
                        const void *v_cache, int dtype, const int32_t *block_tables,
                        const int32_t *context_lens, const int32_t *query_start_loc,
                        int n_chunks, int H_q, int H_kv, int D, int bs, int MB, int64_t NB,
                        double scale, int window, const uint8_t *select)
{
    int rc = check_heads(H_q, H_kv, D, bs, MB, NB);
    if (rc) return rc;
    if (n_chunks < 0 || query_start_loc[0] != 0 || window < 0) return OR_BAD_ARG;
    for (int c = 0; c < n_chunks; ++c) {
        int64_t C = (int64_t)query_start_loc[c + 1] - query_start_loc[c];
        if (C < 0 || context_lens[c] < C || (int64_t)context_lens[c] > (int64_t)MB * bs)
            return OR_BAD_ARG;
    }
    const int64_t total_q = query_start_loc[n_chunks];
    const int group = H_q / H_kv;
    int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 4) reduction(max : err)
    for (int64_t rh = 0; rh < total_q * H_q; ++rh) {
        if (select && !select[rh]) continue;
        int64_t row = rh / H_q;
        int h = (int)(rh % H_q);
        int c = 0;
        while (query_start_loc[c + 1] <= row) ++c;
        int64_t C = (int64_t)query_start_loc[c + 1] - query_start_loc[c];
        int64_t i = row - query_start_loc[c];
        int64_t pos = (int64_t)context_lens[c] - C + i; /* this query's position */
        int64_t j0 = window > 0 && pos + 1 - window > 0 ? pos + 1 - window : 0;
        paged_seq s = {k_cache, v_cache, dtype, block_tables + (int64_t)c * MB, MB,
                       H_kv, D, bs, NB, h / group, 1.0, 1.0};
        double *qv = malloc(sizeof(double) * D);
        double *sbuf = malloc(sizeof(double) * (pos + 1));
        if (!qv || !sbuf) {
            free(qv); free(sbuf);
            err = OR_NO_MEM > err ? OR_NO_MEM : err;
            continue;
        }
        for (int d = 0; d < D; ++d) qv[d] = stored(q, rh * D + d, dtype);
        double l;
        int r = attend(out + rh * D, &l, qv, &s, j0, pos + 1, scale, sbuf);
        if (lse) lse[rh] = l;
        if (r > err) err = r;
        free(qv);
        free(sbuf);
    }
    return err;
}

int oracle_prefill(double *out, double *lse, const void *q, const void *k_cache,
                   const void *v_cache, int dtype, const int32_t *block_tables,
                   const int32_t *context_lens, const int32_t *query_start_loc, int n_chunks,
                   int H_q, int H_kv, int D, int bs, int MB, int64_t NB, double scale,
                   const uint8_t *select)
{
    return prefill_impl(out, lse, q, k_cache, v_cache, dtype, block_tables, context_lens,
                        query_start_loc, n_chunks, H_q, H_kv, D, bs, MB, NB, scale, 0, select);
}

/* [SW]+[CP] chunked prefill with a sliding window: as oracle_prefill, query i
 * (at position pos = ctx - C + i) attending positions
 * [max(0, pos - window + 1), pos] only: the window's last `window` positions
 * end at the query's own, as a decode query at position ctx - 1 attends
 * [ctx - window, ctx). window > 0. */
int oracle_prefill_window(double *out, double *lse, const void *q, const void *k_cache,
                          const void *v_cache, int dtype, const int32_t *block_tables,
                          const int32_t *context_lens, const int32_t *query_start_loc,
                          int n_chunks, int H_q, int H_kv, int D, int bs, int MB, int64_t NB,
                          double scale, int window, const uint8_t *select)
{
    if (window <= 0) return OR_BAD_ARG;
    return prefill_impl(out, lse, q, k_cache, v_cache, dtype, block_tables, context_lens,
                        query_start_loc, n_chunks, H_q, H_kv, D, bs, MB, NB, scale, window,
                        select);
}

/* Block copies of the paged pool, whole blocks (every K/V head) at a time:
 * page "字节跳动 AI Infra (2)", question "vLLM与PagedAttention的原理": a beam
 * that must write into a block it shares gets a copy of it first (B6' is a
 * copy-on-write copy of B6); the scheduler moves a swapped-out request's
 * blocks to CPU memory and back (same page, scheduler section: KV cache
 * swapped to CPU when memory runs short).
 * For each pair i: block mapping[2i+1] of (dst_k, dst_v) := block mapping[2i]
 * of (src_k, src_v); a block is block_bytes contiguous bytes. A pair with an
 * id outside its pool returns OR_BAD_BLOCK before anything is written. */
int oracle_copy_blocks(const void *src_k, const void *src_v, int64_t src_blocks, void *dst_k,
                       void *dst_v, int64_t dst_blocks, const int64_t *mapping, int64_t num_pairs,
                       int64_t block_bytes)
{
    if (num_pairs < 0 || block_bytes <= 0 || src_blocks <= 0 || dst_blocks <= 0) return OR_BAD_ARG;
    for (int64_t i = 0; i < num_pairs; ++i)
        if (mapping[2 * i] < 0 || mapping[2 * i] >= src_blocks || mapping[2 * i + 1] < 0 ||
            mapping[2 * i + 1] >= dst_blocks)
            return OR_BAD_BLOCK;
    for (int64_t i = 0; i < num_pairs; ++i) {
        size_t s = (size_t)mapping[2 * i] * block_bytes, d = (size_t)mapping[2 * i + 1] * block_bytes;
        memcpy((char *)dst_k + d, (const char *)src_k + s, block_bytes);
        memcpy((char *)dst_v + d, (const char *)src_v + s, block_bytes);
    }
    return OR_OK;
}

/* [Q8]+[KV] the append step into an 8-bit cache: each element of the new
 * token's K (V) row for K/V head h is stored as the code of the fp32 quotient
 * x / k_scale[h] (x / v_scale[h]), computed as an IEEE single-precision
 * division and encoded by oracle_e4m3_encode (fmt OR_E4M3) or
 * oracle_int8_encode (fmt OR_I8). key/value are fp32 or bf16 (dtype); caches
 * hold one byte per element. Slots as in oracle_reshape_and_cache. */
static int reshape_q8(const void *key, const void *value, int dtype, uint8_t *k_cache,
                      uint8_t *v_cache, const int64_t *slot_mapping, int64_t num_tokens,
                      int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                      const float *k_scale, const float *v_scale, int fmt)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return OR_BAD_ARG;
    for (int64_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_blocks * (int64_t)block_size) return OR_BAD_SLOT;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / block_size, offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            int64_t dst = ((block * num_kv_heads + h) * block_size + offset) * head_dim;
            for (int d = 0; d < head_dim; ++d) {
                float xk = (float)stored(key, src + d, dtype);
                float xv = (float)stored(value, src + d, dtype);
                float qk = xk / k_scale[h];
                float qv = xv / v_scale[h];
                if (fmt == OR_I8) {
                    k_cache[dst + d] = (uint8_t)oracle_int8_encode(qk);
                    v_cache[dst + d] = (uint8_t)oracle_int8_encode(qv);
                } else {
                    k_cache[dst + d] = oracle_e4m3_encode(qk);
                    v_cache[dst + d] = oracle_e4m3_encode(qv);
                }
            }
        }
    }
    return OR_OK;
}

int oracle_reshape_and_cache_e4m3(const void *key, const void *value, int dtype, uint8_t *k_cache,
                                  uint8_t *v_cache, const int64_t *slot_mapping,
                                  int64_t num_tokens, int num_kv_heads, int head_dim,
                                  int block_size, int64_t num_blocks, const float *k_scale,
                                  const float *v_scale)
{
    return reshape_q8(key, value, dtype, k_cache, v_cache, slot_mapping, num_tokens,
                      num_kv_heads, head_dim, block_size, num_blocks, k_scale, v_scale, OR_E4M3);
}

int oracle_reshape_and_cache_int8(const void *key, const void *value, int dtype, int8_t *k_cache,
                                  int8_t *v_cache, const int64_t *slot_mapping,
                                  int64_t num_tokens, int num_kv_heads, int head_dim,
                                  int block_size, int64_t num_blocks, const float *k_scale,
                                  const float *v_scale)
{
    return reshape_q8(key, value, dtype, (uint8_t *)k_cache, (uint8_t *)v_cache, slot_mapping,
                      num_tokens, num_kv_heads, head_dim, block_size, num_blocks, k_scale,
                      v_scale, OR_I8);
}

/* [KV]+[PG]+[GQA]+[Q8] decode over an 8-bit cache (fmt OR_E4M3 or OR_I8): as
 * oracle_decode, with q of dtype q_dtype and every cached element equal to
 * its code's value times the K/V head's scale (k_scale / v_scale, one per K/V
 * head). */
static int decode_q8(double *out, double *lse, const void *q, int q_dtype, const void *k_cache,
                     const void *v_cache, const float *k_scale, const float *v_scale,
                     const int32_t *block_tables, const int32_t *context_lens, int B, int H_q,
                     int H_kv, int D, int bs, int MB, int64_t NB, double scale,
                     const uint8_t *select, int fmt)
{
    int rc = check_heads(H_q, H_kv, D, bs, MB, NB);
    if (rc) return rc;
    for (int b = 0; b < B; ++b)
        if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs) return OR_BAD_ARG;
    const int group = H_q / H_kv;
    int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : err)
    for (int64_t bh = 0; bh < (int64_t)B * H_q; ++bh) {
        if (select && !select[bh]) continue;
        int b = (int)(bh / H_q), h = (int)(bh % H_q);
        int kvh = h / group;
        paged_seq s = {k_cache, v_cache, fmt, block_tables + (int64_t)b * MB, MB,
                       H_kv, D, bs, NB, kvh, (double)k_scale[kvh], (double)v_scale[kvh]};
        double *qv = malloc(sizeof(double) * D);
        double *sbuf = malloc(sizeof(double) * (context_lens[b] > 0 ? context_lens[b] : 1));
        if (!qv || !sbuf) {
            free(qv); free(sbuf);
            err = OR_NO_MEM > err ? OR_NO_MEM : err;
            continue;
        }
        for (int d = 0; d < D; ++d) qv[d] = stored(q, bh * D + d, q_dtype);
        double l;
        int r = attend(out + bh * D, &l, qv, &s, 0, context_lens[b], scale, sbuf);
        if (lse) lse[bh] = l;
        if (r > err) err = r;
        free(qv);
        free(sbuf);
    }
    return err;
}


int oracle_decode_e4m3(double *out, double *lse, const void *q, int q_dtype, const uint8_t *k_cache,
                       const uint8_t *v_cache, const float *k_scale, const float *v_scale,
                       const int32_t *block_tables, const int32_t *context_lens, int B, int H_q,
                       int H_kv, int D, int bs, int MB, int64_t NB, double scale,
                       const uint8_t *select)
{
    return decode_q8(out, lse, q, q_dtype, k_cache, v_cache, k_scale, v_scale, block_tables,
                     context_lens, B, H_q, H_kv, D, bs, MB, NB, scale, select, OR_E4M3);
}

int oracle_decode_int8(double *out, double *lse, const void *q, int q_dtype, const int8_t *k_cache,
                       const int8_t *v_cache, const float *k_scale, const float *v_scale,
                       const int32_t *block_tables, const int32_t *context_lens, int B, int H_q,
                       int H_kv, int D, int bs, int MB, int64_t NB, double scale,
                       const uint8_t *select)
{
    return decode_q8(out, lse, q, q_dtype, k_cache, v_cache, k_scale, v_scale, block_tables,
                     context_lens, B, H_q, H_kv, D, bs, MB, NB, scale, select, OR_I8);
}

/* [Q8] element-wise helpers over arrays (for tests and fixtures). */
void oracle_int8_encode_array(const float *q, int8_t *codes, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = oracle_int8_encode(q[i]);
}

void oracle_e4m3_encode_array(const float *x, uint8_t *codes, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_array(const uint8_t *codes, double *x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) x[i] = e4m3_value(codes[i]);
}

/* [SW]+[KV]+[PG] decode with a sliding window: as oracle_decode, each query
 * attending positions [max(0, ctx - window), ctx) only (window > 0). */
int oracle_decode_window(double *out, double *lse, const void *q, const void *k_cache,
                         const void *v_cache, int dtype, const int32_t *block_tables,
                         const int32_t *context_lens, int B, int H_q, int H_kv, int D, int bs,
                         int MB, int64_t NB, double scale, int window, const uint8_t *select)
{
    int rc = check_heads(H_q, H_kv, D, bs, MB, NB);
    if (rc) return rc;
    if (window <= 0) return OR_BAD_ARG;
    for (int b = 0; b < B; ++b)
        if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs) return OR_BAD_ARG;
    const int group = H_q / H_kv;
    int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : err)
    for (int64_t bh = 0; bh < (int64_t)B * H_q; ++bh) {
        if (select && !select[bh]) continue;
        int b = (int)(bh / H_q), h = (int)(bh % H_q);
        paged_seq s = {k_cache, v_cache, dtype, block_tables + (int64_t)b * MB, MB,
                       H_kv, D, bs, NB, h / group, 1.0, 1.0};
        int64_t j1 = context_lens[b];
        int64_t j0 = j1 - window > 0 ? j1 - window : 0;
        double *qv = malloc(sizeof(double) * D);
        double *sbuf = malloc(sizeof(double) * (j1 - j0 > 0 ? j1 - j0 : 1));
        if (!qv || !sbuf) {
            free(qv); free(sbuf);
            err = OR_NO_MEM > err ? OR_NO_MEM : err;
            continue;
        }
        for (int d = 0; d < D; ++d) qv[d] = stored(q, bh * D + d, dtype);
        double l;
        int r = attend(out + bh * D, &l, qv, &s, j0, j1, scale, sbuf);
        if (lse) lse[bh] = l;
        if (r > err) err = r;
        free(qv);
        free(sbuf);
    }
    return err;
}

