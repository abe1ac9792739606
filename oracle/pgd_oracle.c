/*
 * pgd_oracle.c -- plain, slow, single-threaded fp64 CPU oracle for paged GQA
 * decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path includes, links or
 * calls this file; it shares no code, header, table or constant with the
 * CUDA library.  Only the test suite, the smoke check and the bench's CPU
 * baseline load it (through ctypes).
 *
 * Sources (the pages this computes from):
 *   [P4-std]  froggydisk, "attention kernels", section "standard attention":
 *             S = Q K^T, P = softmax(S) row-wise, O = P V.
 *   [P4-FA]   same page, section "FlashAttention": online softmax over K blocks
 *             (running max and exponent sum, rescale the accumulated output
 *             when the max changes) gives exactly the full-row result.
 *   [P4-dec]  same page, section "prefill and decode attention": decode splits
 *             the work along the KV length and merges the per-split results
 *             the same way as the online softmax; GQA reuses one KV head for
 *             the several query heads that share it.
 *   [P4-page] same page, section "paged KV and kernels": the kernel reads
 *             K/V through a block table that maps block numbers to addresses.
 *   [P2-3.4]  beengineer500, "batching and attention", section 3.4
 *             (PagedAttention): fixed-size blocks, a block table from logical
 *             to physical block, blocks need not be contiguous.
 *   [P2-2.4]  same page, section 2.4: num_attention_heads / num_key_value_heads;
 *             32 / 8 = 4 query heads share one KV head.
 *   [P4-choose] same page as P4, section "what to check": FP8 KV read directly.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - KV cache layout: [num_blocks][num_kv_heads][block_size][head_dim].
 *   - Query head i uses KV head i / g with g = num_q_heads / num_kv_heads.
 *   - Token t of sequence s lives in physical block block_table[s][t / bs]
 *     at offset t % bs.
 *   - A context of length 0 gives out = 0 and lse = -inf.
 *   - FP8 E4M3 values are byte -> e4m3 value (bias 7, subnormals m * 2^-9,
 *     0x7F / 0xFF NaN, no infinity) times a per-KV-head fp32 scale.
 *   - kv_append: a slot below zero is a padding token and is skipped.
 *   - The split merge is the log-sum-exp weighting of the per-split
 *     (normalised output, lse) pairs.
 *
 * Every floating-point step is fp64; sums run in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PGDO_OK 0
#define PGDO_EINVAL 1

/* KV element formats understood by the oracle. */
#define PGDO_BF16 0
#define PGDO_E4M3 1

/* ------------------------------------------------------------------------- */
/* Number formats, written from their definitions.                           */
/* ------------------------------------------------------------------------- */

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 mantissa bits. */
double pgdo_bf16_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 7) & 0xFF;
    int man = bits & 0x7F;
    double mag;
    if (expo == 0) {
        mag = ldexp((double)man, -126 - 7);          /* subnormal */
    } else if (expo == 0xFF) {
        mag = man ? NAN : INFINITY;
    } else {
        mag = ldexp(1.0 + (double)man / 128.0, expo - 127);
    }
    return sign ? -mag : mag;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; there is
 * no infinity; the largest finite magnitude is 1.75 * 2^8 = 448. */
double pgdo_e4m3_to_double(uint8_t bits)
{
    int sign = (bits >> 7) & 1;
    int expo = (bits >> 3) & 0xF;
    int man = bits & 0x7;
    double mag;
    if (expo == 0xF && man == 0x7) {
        mag = NAN;
    } else if (expo == 0) {
        mag = ldexp((double)man, -9);
    } else {
        mag = ldexp(1.0 + (double)man / 8.0, expo - 7);
    }
    return sign ? -mag : mag;
}

/* Nearest E4M3 value to y, ties to the even mantissa, magnitudes above the
 * largest finite value (448) saturating to +-448 and NaN giving 0x7F.  Written
 * from the format: normal values (1 + m/8) * 2^(e-7) for e = 1..15 (S.1111.111
 * excluded), subnormals m * 2^-9.  The default floating-point rounding mode
 * (to nearest, ties to even) makes nearbyint the tie-to-even step. */
uint8_t pgdo_e4m3_from_double(double y)
{
    if (isnan(y)) return 0x7F;
    const int sign = signbit(y) ? 0x80 : 0;
    const double a = fabs(y);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {                      /* subnormal range */
        const int k = (int)nearbyint(ldexp(a, 9));  /* a / 2^-9, 0..8 */
        return (uint8_t)(sign | (k == 8 ? 0x08 : k)); /* 8 * 2^-9 is the smallest normal */
    }
    int e2;
    frexp(a, &e2);                                 /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                                /* a in [2^E, 2^(E+1)) */
    int m = (int)nearbyint((ldexp(a, -E) - 1.0) * 8.0);
    if (m == 8) { m = 0; ++E; }
    if (E > 8 || (E == 8 && m == 7)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | ((E + 7) << 3) | m);
}

void pgdo_encode_e4m3_array(const double *src, uint8_t *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = pgdo_e4m3_from_double(src[i]);
}

void pgdo_decode_bf16_array(const uint16_t *src, double *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = pgdo_bf16_to_double(src[i]);
}

void pgdo_decode_e4m3_array(const uint8_t *src, double *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = pgdo_e4m3_to_double(src[i]);
}

/* ------------------------------------------------------------------------- */
/* KV append: copy each new token's K and V rows into its cache slot.        */
/* [P2-3.4] fixed-size blocks; slot = physical_block * block_size + offset.  */
/* ------------------------------------------------------------------------- */
int pgdo_kv_append(const void *k_new, const void *v_new,
                   const int64_t *slot_mapping, int32_t num_tokens,
                   void *k_cache, void *v_cache,
                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                   int32_t num_blocks, int32_t elem_bytes)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks < 0 || (elem_bytes != 1 && elem_bytes != 2))
        return PGDO_EINVAL;
    const int64_t row = (int64_t)head_dim * elem_bytes;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;                           /* padding token */
        if (slot >= (int64_t)num_blocks * block_size) return PGDO_EINVAL;
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)t * num_kv_heads + h) * row;
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * row;
            memcpy((char *)k_cache + dst, (const char *)k_new + src, (size_t)row);
            memcpy((char *)v_cache + dst, (const char *)v_new + src, (size_t)row);
        }
    }
    return PGDO_OK;
}

/* ------------------------------------------------------------------------- */
/* Quantising KV append: bf16 K/V rows of new tokens go into an FP8 E4M3     */
/* cache ("attention kernels", "what to check": FP8 KV cache).  Each element */
/* is divided by its KV head's fp32 scale in fp32 (the precision the kernel  */
/* decides the code in), then rounded to the nearest E4M3 value (ties to     */
/* even, saturating at +-448) by pgdo_e4m3_from_double.                      */
/* ------------------------------------------------------------------------- */
int pgdo_kv_append_quant(const uint16_t *k_new, const uint16_t *v_new,
                         const int64_t *slot_mapping, int32_t num_tokens,
                         uint8_t *k_cache, uint8_t *v_cache,
                         const float *k_scale, const float *v_scale,
                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         int32_t num_blocks)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks < 0 || !k_scale || !v_scale)
        return PGDO_EINVAL;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) return PGDO_EINVAL;
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) {
                float kx = (float)pgdo_bf16_to_double(k_new[src + d]);
                float vx = (float)pgdo_bf16_to_double(v_new[src + d]);
                float ky = kx / k_scale[h];
                float vy = vx / v_scale[h];
                k_cache[dst + d] = pgdo_e4m3_from_double((double)ky);
                v_cache[dst + d] = pgdo_e4m3_from_double((double)vy);
            }
        }
    }
    return PGDO_OK;
}

/* ------------------------------------------------------------------------- */
/* Shared argument block for the attention functions.                        */
/* ------------------------------------------------------------------------- */
typedef struct {
    const uint16_t *q;          /* bf16 [num_seqs][num_q_heads][head_dim]      */
    const void *k_cache;        /* [num_blocks][num_kv_heads][block_size][D]   */
    const void *v_cache;
    int kv_dtype;               /* PGDO_BF16 or PGDO_E4M3                      */
    const float *k_scale;       /* [num_kv_heads], FP8 only                    */
    const float *v_scale;
    const int32_t *block_table; /* [num_seqs][max_blocks_per_seq]              */
    int32_t max_blocks_per_seq;
    const int32_t *context_lens;
    int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks;
    double scale;
    int32_t window;             /* > 0: attend to the last `window` tokens only */
} pgdo_args;

static int check_args(const pgdo_args *a)
{
    if (!a->q || !a->k_cache || !a->v_cache || !a->block_table || !a->context_lens)
        return PGDO_EINVAL;
    if (a->num_seqs < 0 || a->num_q_heads <= 0 || a->num_kv_heads <= 0 ||
        a->head_dim <= 0 || a->block_size <= 0 || a->num_blocks < 0 ||
        a->max_blocks_per_seq < 0)
        return PGDO_EINVAL;
    if (a->num_q_heads % a->num_kv_heads) return PGDO_EINVAL;
    if (a->kv_dtype != PGDO_BF16 && a->kv_dtype != PGDO_E4M3) return PGDO_EINVAL;
    if (a->kv_dtype == PGDO_E4M3 && (!a->k_scale || !a->v_scale)) return PGDO_EINVAL;
    for (int32_t s = 0; s < a->num_seqs; ++s) {
        int32_t n = a->context_lens[s];
        if (n < 0 || n > (int64_t)a->max_blocks_per_seq * a->block_size) return PGDO_EINVAL;
        for (int32_t j = 0; j < (n + a->block_size - 1) / a->block_size; ++j) {
            int32_t pb = a->block_table[(int64_t)s * a->max_blocks_per_seq + j];
            if (pb < 0 || pb >= a->num_blocks) return PGDO_EINVAL;
        }
    }
    return PGDO_OK;
}

/* Gather one cached row (K or V) of token t of sequence s, KV head h, and
 * decode it to fp64.  [P2-3.4], [P4-page]: logical block t / bs is looked up
 * in the block table; the token sits at offset t % bs inside that block. */
static void gather_row(const pgdo_args *a, const void *cache, const float *scales,
                       int32_t s, int32_t h, int32_t t, double *row)
{
    int32_t pb = a->block_table[(int64_t)s * a->max_blocks_per_seq + t / a->block_size];
    int32_t off = t % a->block_size;
    int64_t base = (((int64_t)pb * a->num_kv_heads + h) * a->block_size + off) * a->head_dim;
    if (a->kv_dtype == PGDO_BF16) {
        const uint16_t *c = (const uint16_t *)cache;
        for (int32_t d = 0; d < a->head_dim; ++d) row[d] = pgdo_bf16_to_double(c[base + d]);
    } else {
        const uint8_t *c = (const uint8_t *)cache;
        double sc = (double)scales[h];
        for (int32_t d = 0; d < a->head_dim; ++d) row[d] = pgdo_e4m3_to_double(c[base + d]) * sc;
    }
}

/* Query row of head i of sequence s, decoded to fp64. */
static void load_q(const pgdo_args *a, int32_t s, int32_t i, double *qrow)
{
    const uint16_t *q = a->q + ((int64_t)s * a->num_q_heads + i) * a->head_dim;
    for (int32_t d = 0; d < a->head_dim; ++d) qrow[d] = pgdo_bf16_to_double(q[d]);
}

/* Score of one key: x = scale * sum_d q_d k_d, summed in order d = 0..D-1.
 * [P4-std] S = Q K^T, with the softmax scale applied to the scores. */
static double score(const double *qrow, const double *krow, int32_t D, double scale)
{
    double acc = 0.0;
    for (int32_t d = 0; d < D; ++d) acc += qrow[d] * krow[d];
    return scale * acc;
}

/* ------------------------------------------------------------------------- */
/* The plain definition, one (sequence, query head) row at a time.           */
/* [P4-std]: S = Q K^T, P = softmax(S), O = P V, for a single query row.     */
/* [P4-dec] / [P2-2.4]: query head i reads KV head i / g.                    */
/* With a window W > 0 (sliding-window attention: the co-design page's       */
/* principle 3 and "batching and attention" 2.3 name it as a way to cut the  */
/* KV state read), the query at position n-1 sees tokens n-W .. n-1 only.    */
/* ------------------------------------------------------------------------- */
/* One query row q (bf16) of sequence s against KV head h over tokens
 * lo .. n-1; an empty range gives out = 0, lse = -inf. */
static void attend(const pgdo_args *a, int32_t s, int32_t h, const uint16_t *q, int32_t lo,
                   int32_t n, double *out, double *lse)
{
    const int32_t D = a->head_dim;
    if (n <= lo) {
        for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double *qrow = malloc(sizeof(double) * D);
    double *row = malloc(sizeof(double) * D);
    double *x = malloc(sizeof(double) * n);
    for (int32_t d = 0; d < D; ++d) qrow[d] = pgdo_bf16_to_double(q[d]);
    /* 1. all scores of the row */
    for (int32_t t = lo; t < n; ++t) {
        gather_row(a, a->k_cache, a->k_scale, s, h, t, row);
        x[t] = score(qrow, row, D, a->scale);
    }
    /* 2. softmax over the whole row: max, exponentials, sum */
    double M = x[lo];
    for (int32_t t = lo + 1; t < n; ++t) if (x[t] > M) M = x[t];
    double Z = 0.0;
    for (int32_t t = lo; t < n; ++t) { x[t] = exp(x[t] - M); Z += x[t]; }
    /* 3. O = P V */
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    for (int32_t t = lo; t < n; ++t) {
        gather_row(a, a->v_cache, a->v_scale, s, h, t, row);
        for (int32_t d = 0; d < D; ++d) out[d] += x[t] * row[d];
    }
    for (int32_t d = 0; d < D; ++d) out[d] /= Z;
    *lse = M + log(Z);
    free(qrow); free(row); free(x);
}

static void plain_row(const pgdo_args *a, int32_t s, int32_t i, double *out, double *lse)
{
    const int32_t g = a->num_q_heads / a->num_kv_heads;
    const int32_t h = i / g;
    const int32_t n = a->context_lens[s];
    const int32_t lo = (a->window > 0 && n > a->window) ? n - a->window : 0;
    attend(a, s, h, a->q + ((int64_t)s * a->num_q_heads + i) * a->head_dim, lo, n, out, lse);
}

#define ARGS_INIT                                                                \
    pgdo_args a = {q, k_cache, v_cache, kv_dtype, k_scale, v_scale, block_table, \
                   max_blocks_per_seq, context_lens, num_seqs, num_q_heads,      \
                   num_kv_heads, head_dim, block_size, num_blocks, scale, 0}

#define ARGS_DECL                                                                     \
    const uint16_t *q, const void *k_cache, const void *v_cache, int32_t kv_dtype,    \
    const float *k_scale, const float *v_scale, const int32_t *block_table,           \
    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,        \
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,  \
    int32_t num_blocks, double scale

/* Whole batch by the plain definition: out fp64 [num_seqs][num_q_heads][D],
 * lse fp64 [num_seqs][num_q_heads] (natural log). */
int pgdo_paged_decode(ARGS_DECL, double *out, double *lse)
{
    ARGS_INIT;
    int rc = check_args(&a);
    if (rc) return rc;
    for (int32_t s = 0; s < num_seqs; ++s)
        for (int32_t i = 0; i < num_q_heads; ++i) {
            int64_t r = (int64_t)s * num_q_heads + i;
            plain_row(&a, s, i, out + r * head_dim, lse + r);
        }
    return PGDO_OK;
}

/* Several query tokens per sequence (speculative-decoding verification, the
 * lecture's section on it; prefill chunks that read a long prefix, the
 * co-design page's agent section): q [num_seqs][q_len][num_q_heads][D]; the
 * q_len newest tokens of sequence s sit at positions n-q_len .. n-1 (n =
 * context_lens[s], which counts them), so query token i sees tokens below
 * n - q_len + 1 + i (causal), and with window W > 0 only the last W of those.
 * out [num_seqs][q_len][num_q_heads][D], lse [num_seqs][q_len][num_q_heads]. */
int pgdo_paged_decode_multi(ARGS_DECL, int32_t q_len, int32_t window, double *out,
                            double *lse)
{
    ARGS_INIT;
    if (q_len < 1 || window < 0) return PGDO_EINVAL;
    int rc = check_args(&a);
    if (rc) return rc;
    const int32_t g = num_q_heads / num_kv_heads;
    for (int32_t s = 0; s < num_seqs; ++s)
        for (int32_t it = 0; it < q_len; ++it)
            for (int32_t i = 0; i < num_q_heads; ++i) {
                const int64_t r = ((int64_t)s * q_len + it) * num_q_heads + i;
                int32_t hi = context_lens[s] - q_len + 1 + it;
                if (hi < 0) hi = 0;
                const int32_t lo = (window > 0 && hi > window) ? hi - window : 0;
                attend(&a, s, i / g, q + r * head_dim, lo, hi, out + r * head_dim, lse + r);
            }
    return PGDO_OK;
}

/* Whole batch with a sliding window of `window` tokens (0 = the full
 * context): query row of sequence s sees tokens max(0, n-W) .. n-1. */
int pgdo_paged_decode_window(ARGS_DECL, int32_t window, double *out, double *lse)
{
    ARGS_INIT;
    int rc = check_args(&a);
    if (rc) return rc;
    if (window < 0) return PGDO_EINVAL;
    a.window = window;
    for (int32_t s = 0; s < num_seqs; ++s)
        for (int32_t i = 0; i < num_q_heads; ++i) {
            int64_t r = (int64_t)s * num_q_heads + i;
            plain_row(&a, s, i, out + r * head_dim, lse + r);
        }
    return PGDO_OK;
}

/* Selected rows only (for sampling full-size workloads): row r is
 * (rows_seq[r], rows_head[r]); out fp64 [n_rows][D], lse fp64 [n_rows]. */
int pgdo_paged_decode_rows(ARGS_DECL, const int32_t *rows_seq, const int32_t *rows_head,
                           int32_t n_rows, double *out, double *lse)
{
    ARGS_INIT;
    if (!rows_seq || !rows_head || n_rows < 0) return PGDO_EINVAL;
    for (int32_t r = 0; r < n_rows; ++r)
        if (rows_seq[r] < 0 || rows_seq[r] >= num_seqs || rows_head[r] < 0 ||
            rows_head[r] >= num_q_heads)
            return PGDO_EINVAL;
    /* Validate only the sequences asked for, so a sample stays cheap. */
    pgdo_args sub = a;
    for (int32_t r = 0; r < n_rows; ++r) {
        sub.num_seqs = 1;
        sub.block_table = a.block_table + (int64_t)rows_seq[r] * max_blocks_per_seq;
        sub.context_lens = a.context_lens + rows_seq[r];
        sub.q = a.q + (int64_t)rows_seq[r] * num_q_heads * head_dim;
        int rc = check_args(&sub);
        if (rc) return rc;
        plain_row(&sub, 0, rows_head[r], out + (int64_t)r * head_dim, lse + r);
    }
    return PGDO_OK;
}

/* ------------------------------------------------------------------------- */
/* Log-sum-exp merge of per-split results.  [P4-dec]: the per-split results  */
/* are combined the same way the online softmax combines blocks.  Each split */
/* p carries its normalised output o_p and lse_p = m_p + ln l_p; then        */
/*   M = max_p lse_p,  w_p = exp(lse_p - M),                                 */
/*   out = sum_p w_p o_p / sum_p w_p,  lse = M + ln sum_p w_p.               */
/* Splits with lse_p = -inf (no tokens) carry no weight.                     */
/* o_part fp64 [num_parts][rows][D]; lse_part fp64 [num_parts][rows].        */
/* ------------------------------------------------------------------------- */
int pgdo_merge_partials(const double *o_part, const double *lse_part, int32_t num_parts,
                        int32_t rows, int32_t head_dim, double *out, double *lse)
{
    if (num_parts < 0 || rows < 0 || head_dim <= 0) return PGDO_EINVAL;
    for (int32_t r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int32_t p = 0; p < num_parts; ++p) {
            double l = lse_part[(int64_t)p * rows + r];
            if (l > M) M = l;
        }
        double *o = out + (int64_t)r * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
        if (M == -INFINITY) { lse[r] = -INFINITY; continue; }
        double W = 0.0;
        for (int32_t p = 0; p < num_parts; ++p) {
            double l = lse_part[(int64_t)p * rows + r];
            if (l == -INFINITY) continue;
            double w = exp(l - M);
            W += w;
            const double *op = o_part + ((int64_t)p * rows + r) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) o[d] += w * op[d];
        }
        for (int32_t d = 0; d < head_dim; ++d) o[d] /= W;
        lse[r] = M + log(W);
    }
    return PGDO_OK;
}

/* ------------------------------------------------------------------------- */
/* Second, independent route to the same numbers: the row is cut into       */
/* partitions of partition_tokens tokens; inside each partition the keys are */
/* visited in tiles of tile_tokens with the online softmax of [P4-FA]        */
/* (running max m, running sum l, accumulated output rescaled by             */
/* exp(m_old - m_new) when the max grows); the partitions are then merged by */
/* pgdo_merge_partials ([P4-dec]).  Used to pin that tiling, splitting and   */
/* merging leave the plain result unchanged.                                 */
/* ------------------------------------------------------------------------- */
static void tiled_row(const pgdo_args *a, int32_t s, int32_t i, int32_t tile_tokens,
                      int32_t partition_tokens, double *out, double *lse)
{
    const int32_t D = a->head_dim;
    const int32_t g = a->num_q_heads / a->num_kv_heads;
    const int32_t h = i / g;
    const int32_t n = a->context_lens[s];
    const int32_t P = n == 0 ? 0 : (n + partition_tokens - 1) / partition_tokens;
    double *qrow = malloc(sizeof(double) * D);
    double *row = malloc(sizeof(double) * D);
    double *xt = malloc(sizeof(double) * tile_tokens);
    double *o_part = calloc((size_t)(P ? P : 1) * D, sizeof(double));
    double *lse_part = malloc(sizeof(double) * (P ? P : 1));
    load_q(a, s, i, qrow);
    for (int32_t p = 0; p < P; ++p) {
        int32_t t0 = p * partition_tokens;
        int32_t t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n;
        double m = -INFINITY, l = 0.0;
        double *acc = o_part + (int64_t)p * D;        /* zero-initialised */
        for (int32_t u0 = t0; u0 < t1; u0 += tile_tokens) {
            int32_t u1 = u0 + tile_tokens < t1 ? u0 + tile_tokens : t1;
            double m_tile = -INFINITY;
            for (int32_t t = u0; t < u1; ++t) {
                gather_row(a, a->k_cache, a->k_scale, s, h, t, row);
                xt[t - u0] = score(qrow, row, D, a->scale);
                if (xt[t - u0] > m_tile) m_tile = xt[t - u0];
            }
            double m_new = m > m_tile ? m : m_tile;
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            l *= alpha;
            for (int32_t d = 0; d < D; ++d) acc[d] *= alpha;
            for (int32_t t = u0; t < u1; ++t) {
                double w = exp(xt[t - u0] - m_new);
                l += w;
                gather_row(a, a->v_cache, a->v_scale, s, h, t, row);
                for (int32_t d = 0; d < D; ++d) acc[d] += w * row[d];
            }
            m = m_new;
        }
        for (int32_t d = 0; d < D; ++d) acc[d] /= l;
        lse_part[p] = m + log(l);
    }
    pgdo_merge_partials(o_part, lse_part, P, 1, D, out, lse);
    free(qrow); free(row); free(xt); free(o_part); free(lse_part);
}

int pgdo_paged_decode_tiled(ARGS_DECL, int32_t tile_tokens, int32_t partition_tokens,
                            double *out, double *lse)
{
    ARGS_INIT;
    int rc = check_args(&a);
    if (rc) return rc;
    if (tile_tokens <= 0 || partition_tokens <= 0) return PGDO_EINVAL;
    for (int32_t s = 0; s < num_seqs; ++s)
        for (int32_t i = 0; i < num_q_heads; ++i) {
            int64_t r = (int64_t)s * num_q_heads + i;
            tiled_row(&a, s, i, tile_tokens, partition_tokens, out + r * head_dim, lse + r);
        }
    return PGDO_OK;
}
