/*
 * csa2_ref.c -- plain, slow CPU oracle for the CSA2 decode step over an FP4
 * global KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library: every number format and
 * every step below is written out again from its definition.
 *
 * Sources (web pages on "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache
 * Compression"):
 *   [TLDR]   tldrocket.com retelling of the MarkTechPost piece, paragraph 3
 *            ("Full, Reindex, or Reuse roles"; candidate pool of up to
 *            16,384 positions) and paragraph 4 (main KV quantised to E2M1
 *            with one E4M3 scale per 16 channels, NVFP4 without the global
 *            scale); paragraph 2 (sliding window in every layer, 128 tokens).
 *   [HN]     hackernews.kjhq.dev post 49735410, key points 2 and 3 (layers
 *            share the same main KV and Top-K indices; hierarchical sparse
 *            indexer with a shallow-layer candidate pool).
 *   [FANOUT] fanout.sh daily lesson, "What you will learn", item 2 (modes
 *            share global KV and sparse selections, keep layer-local queries).
 *
 * Readings taken where the pages are silent (each one is listed with its
 * justification in the design notes of the repository):
 *   - scoring function: s_t = sum_h w_h * max(0, q_h . k_t)   (pages give none)
 *   - one cache entry per token; one latent per position serves as key and
 *     value for every head; one index key per position shared by all layers
 *   - block scale s = E4M3_RNE_satfinite(fp32(amax / 6)), codes
 *     c_i = E2M1_RNE_satfinite(fp32(x_i / s)); s == 0 gives all-zero codes
 *   - attention set S = window ∪ top-k, window = [max(0,p-W+1), p]
 *   - ties in selection: score descending, then position ascending
 *
 * Everything that is not the exact fp32 quantisation runs in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define REF_OK 0
#define REF_ERR_ARG 1
#define REF_ERR_BOUNDS 5

#define REF_F32 0
#define REF_BF16 1
#define REF_E4M3 2

/* ------------------------------------------------------------------------ */
/* Number formats.  [TLDR] paragraph 4 names E2M1 codes with E4M3 scales     */
/* ("NVFP4 without the global scale").                                      */
/* ------------------------------------------------------------------------ */

/* E4M3 (finite variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent field 0 is subnormal (2^-6 * m/8); S.1111.111 is NaN and
 * there is no infinity, so the largest finite magnitude is 2^8 * 1.75 = 448. */
double ref_e4m3_value(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 7;
    double mag;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, 1 - 7);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* E2M1: 1 sign bit (bit 3), 2 exponent bits with bias 1, 1 mantissa bit;
 * exponent field 0 is subnormal (m * 0.5); no infinity, no NaN. */
double ref_e2m1_value(uint8_t c)
{
    int sign = (c >> 3) & 1;
    int e = (c >> 1) & 3;
    int m = c & 1;
    double mag;
    if (e == 0)
        mag = ldexp((double)m / 2.0, 1 - 1);
    else
        mag = ldexp(1.0 + (double)m / 2.0, e - 1);
    return sign ? -mag : mag;
}

/* Round-to-nearest-even with saturation to the largest finite magnitude.
 * The non-negative codes 0..top have strictly increasing values; pick the one
 * nearest to |x|, and on an exact tie between two neighbouring codes the one
 * with an even code (even mantissa).  |x| at or beyond the top value stays on
 * the top code (saturation).  The sign of x is kept, so a negative value that
 * rounds to zero encodes as negative zero.  x must be finite. */
static int nearest_code(double a, double (*value)(uint8_t), int top)
{
    int lo = 0, hi = top;          /* last code whose value is <= a */
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (value((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
    }
    if (lo == top) return top;
    double d0 = a - value((uint8_t)lo);
    double d1 = value((uint8_t)(lo + 1)) - a;
    if (d1 < d0 || (d1 == d0 && ((lo + 1) & 1) == 0)) return lo + 1;
    return lo;
}

uint8_t ref_e4m3_encode(float xf)
{
    double x = (double)xf;
    int code = nearest_code(fabs(x), ref_e4m3_value, 0x7E);
    return (uint8_t)((signbit(x) ? 0x80 : 0) | code);
}

uint8_t ref_e2m1_encode(float xf)
{
    double x = (double)xf;
    int code = nearest_code(fabs(x), ref_e2m1_value, 7);
    return (uint8_t)((signbit(x) ? 8 : 0) | code);
}

int ref_e2m1_encode_array(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        if (!isfinite(x[i])) return REF_ERR_ARG;
        out[i] = ref_e2m1_encode(x[i]);
    }
    return REF_OK;
}

/* bfloat16 is the top half of an IEEE binary32 word. */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static double load_value(int dtype, const void* base, int64_t i)
{
    if (dtype == REF_F32) return (double)((const float*)base)[i];
    if (dtype == REF_BF16) return (double)bf16_to_f32(((const uint16_t*)base)[i]);
    return ref_e4m3_value(((const uint8_t*)base)[i]);
}

/* ------------------------------------------------------------------------ */
/* Block quantisation of one 16-channel block ([TLDR] paragraph 4).          */
/*   amax = max_i |x_i|            (bf16 inputs widened exactly to fp32)     */
/*   s    = E4M3(fp32(amax / 6))   (6 is the largest E2M1 magnitude)         */
/*   c_i  = E2M1(fp32(x_i / s)),   all codes 0 when s decodes to 0           */
/* Divisions are IEEE binary32 divisions, as the fp32 steps are the reading. */
/* Returns REF_ERR_ARG on a non-finite input.                                */
/* ------------------------------------------------------------------------ */
int ref_quantize_block16(const float* x, uint8_t* codes, uint8_t* scale)
{
    volatile float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        if (!isfinite(x[i])) return REF_ERR_ARG;
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    volatile float six = 6.0f;
    volatile float sf = amax / six;
    uint8_t sc = ref_e4m3_encode(sf);
    volatile float s = (float)ref_e4m3_value(sc);
    *scale = sc;
    for (int i = 0; i < 16; ++i) {
        if (s == 0.0f) {
            codes[i] = 0;
        } else {
            volatile float q = x[i] / s;
            codes[i] = ref_e2m1_encode(q);
        }
    }
    return REF_OK;
}

/* One FP4 row: D/2 code bytes (channel 2j in the low nibble of byte j, channel
 * 2j+1 in the high nibble) followed by D/16 E4M3 scale bytes; the rest of the
 * row_stride bytes are left untouched. */
int ref_quantize_row(const uint16_t* x_bf16, int D, uint8_t* row)
{
    if (D <= 0 || D % 16) return REF_ERR_ARG;
    for (int blk = 0; blk < D / 16; ++blk) {
        float x[16];
        uint8_t codes[16], sc;
        for (int i = 0; i < 16; ++i) x[i] = bf16_to_f32(x_bf16[blk * 16 + i]);
        int rc = ref_quantize_block16(x, codes, &sc);
        if (rc) return rc;
        for (int j = 0; j < 8; ++j)
            row[blk * 8 + j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
        row[D / 2 + blk] = sc;
    }
    return REF_OK;
}

int ref_quantize_rows(const uint16_t* x_bf16, int64_t n, int D, int row_stride, uint8_t* rows)
{
    if (row_stride < D / 2 + D / 16) return REF_ERR_ARG;
    for (int64_t r = 0; r < n; ++r) {
        int rc = ref_quantize_row(x_bf16 + r * D, D, rows + r * row_stride);
        if (rc) return rc;
    }
    return REF_OK;
}

/* dequant(c, s) = value(c) * value(s), exact in fp64. */
int ref_dequant_row(const uint8_t* row, int D, double* out)
{
    if (D <= 0 || D % 16) return REF_ERR_ARG;
    for (int d = 0; d < D; ++d) {
        uint8_t byte = row[d / 2];
        uint8_t code = (d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
        double s = ref_e4m3_value(row[D / 2 + d / 16]);
        out[d] = ref_e2m1_value(code) * s;
    }
    return REF_OK;
}

/* Index keys: E4M3_RNE_satfinite of each (bf16 or fp32) input value. */
int ref_encode_e4m3_array(int src_dtype, const void* src, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        float v = (src_dtype == REF_F32) ? ((const float*)src)[i]
                                         : bf16_to_f32(((const uint16_t*)src)[i]);
        if (!isfinite(v)) return REF_ERR_ARG;
        out[i] = ref_e4m3_encode(v);
    }
    return REF_OK;
}

/* ------------------------------------------------------------------------ */
/* Cache view.  One entry per token; one latent row per position shared by   */
/* all heads as key and value and by all layers ([HN] key point 2); one      */
/* index key per position.  Paged mode: slot = page_table[b][t / page_size]  */
/* * page_size + t % page_size; contiguous mode: slot = b * seq_stride + t.  */
/* ------------------------------------------------------------------------ */
typedef struct {
    uint8_t* rows;            /* [n_slots][row_stride] */
    void* idx_keys;           /* [n_slots][idx_dim] of idx_key_dtype */
    const int32_t* page_table;/* [batch][max_pages] or NULL */
    const int32_t* seq_lens;  /* [batch] */
    int32_t batch, max_pages, page_size, dim, idx_dim, row_stride;
    int64_t seq_stride_slots;
    int64_t n_slots;
    int32_t idx_key_dtype;    /* REF_F32 or REF_E4M3 */
} ref_cache;

int64_t ref_slot(const ref_cache* c, int b, int64_t t)
{
    if (b < 0 || b >= c->batch || t < 0) return -1;
    int64_t slot;
    if (c->page_table) {
        int64_t page = t / c->page_size;
        if (page >= c->max_pages) return -1;
        int32_t phys = c->page_table[(int64_t)b * c->max_pages + page];
        if (phys < 0) return -1;
        slot = (int64_t)phys * c->page_size + t % c->page_size;
    } else {
        if (t >= c->seq_stride_slots) return -1;
        slot = (int64_t)b * c->seq_stride_slots + t;
    }
    if (slot >= c->n_slots) return -1;
    return slot;
}

/* Write n consecutive positions t0.. of sequence b: latent rows x (bf16,
 * [n][dim], nullable) are quantised into FP4 rows; index-key inputs idx
 * (bf16 or fp32, [n][idx_dim], nullable) are stored as E4M3 or fp32 as the
 * cache says. */
int ref_kv_write(const ref_cache* c, int b, int64_t t0, int64_t n, const uint16_t* x, int idx_src_dtype,
                 const void* idx)
{
    for (int64_t i = 0; i < n; ++i) {
        int64_t slot = ref_slot(c, b, t0 + i);
        if (slot < 0) return REF_ERR_BOUNDS;
        if (x) {
            int rc = ref_quantize_row(x + i * c->dim, c->dim, c->rows + slot * c->row_stride);
            if (rc) return rc;
        }
        if (idx) {
            for (int d = 0; d < c->idx_dim; ++d) {
                int64_t src = i * c->idx_dim + d;
                float v = (idx_src_dtype == REF_F32) ? ((const float*)idx)[src]
                                                     : bf16_to_f32(((const uint16_t*)idx)[src]);
                if (!isfinite(v)) return REF_ERR_ARG;
                if (c->idx_key_dtype == REF_E4M3)
                    ((uint8_t*)c->idx_keys)[slot * c->idx_dim + d] = ref_e4m3_encode(v);
                else
                    ((float*)c->idx_keys)[slot * c->idx_dim + d] = v;
            }
        }
    }
    return REF_OK;
}

/* Quantise-on-append: rows x[b][i] (bf16, D channels) land at position
 * start_pos[b] + i of sequence b, for every sequence of the batch. */
int ref_kv_append(const ref_cache* c, const uint16_t* x, int idx_src_dtype, const void* idx_new,
                  const int32_t* start_pos, int n_new)
{
    for (int b = 0; b < c->batch; ++b) {
        const uint16_t* xb = x + (int64_t)b * n_new * c->dim;
        const void* ib = NULL;
        if (idx_new) {
            size_t esz = (idx_src_dtype == REF_F32) ? 4 : 2;
            ib = (const char*)idx_new + (size_t)b * n_new * c->idx_dim * esz;
        }
        int rc = ref_kv_write(c, b, start_pos[b], n_new, xb, idx_src_dtype, ib);
        if (rc) return rc;
    }
    return REF_OK;
}

/* ------------------------------------------------------------------------ */
/* Indexer scoring (reading of [TLDR] paragraph 3 / [HN] key point 3; the     */
/* pages do not give the function):                                          */
/*     s_t = sum_h w_h * max(0, sum_d q[h][d] * k_t[d])                      */
/* computed in fp64 from the stored key values and the given query values.   */
/* positions[i] (or i when positions is NULL) are sequence positions of b.   */
/* ------------------------------------------------------------------------ */
int ref_index_scores(const ref_cache* c, int b, int64_t n, const int32_t* positions,
                     int q_dtype, const void* q, int H_I, const float* w, double* scores)
{
    int Dk = c->idx_dim;
    double* qd = (double*)malloc(sizeof(double) * (size_t)H_I * Dk);
    double* kd = (double*)malloc(sizeof(double) * (size_t)Dk);
    if (!qd || !kd) { free(qd); free(kd); return REF_ERR_ARG; }
    for (int64_t i = 0; i < (int64_t)H_I * Dk; ++i) qd[i] = load_value(q_dtype, q, i);
    int rc = REF_OK;
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = positions ? positions[i] : i;
        int64_t slot = ref_slot(c, b, t);
        if (slot < 0) { rc = REF_ERR_BOUNDS; break; }
        for (int d = 0; d < Dk; ++d) kd[d] = load_value(c->idx_key_dtype, c->idx_keys, slot * Dk + d);
        double s = 0.0;
        for (int h = 0; h < H_I; ++h) {
            double dot = 0.0;
            for (int d = 0; d < Dk; ++d) dot += qd[(int64_t)h * Dk + d] * kd[d];
            s += (double)w[h] * (dot > 0.0 ? dot : 0.0);
        }
        scores[i] = s;
    }
    free(qd);
    free(kd);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Top-n selection: order by score descending, ties by position ascending,   */
/* keep the first min(n_out, n); the rest of out_idx is -1.                  */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int32_t pos; } ref_pair;

static int pair_cmp(const void* a, const void* b)
{
    const ref_pair* x = (const ref_pair*)a;
    const ref_pair* y = (const ref_pair*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

int ref_select_top(const double* scores, const int32_t* positions, int64_t n, int n_out, int32_t* out_idx)
{
    ref_pair* p = (ref_pair*)malloc(sizeof(ref_pair) * (size_t)(n > 0 ? n : 1));
    if (!p) return REF_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        p[i].s = scores[i];
        p[i].pos = positions ? positions[i] : (int32_t)i;
    }
    qsort(p, (size_t)n, sizeof(ref_pair), pair_cmp);
    for (int i = 0; i < n_out; ++i) out_idx[i] = (i < n) ? p[i].pos : -1;
    free(p);
    return REF_OK;
}

/* Query token j of T sits at position p_j = L_b - T + j and sees t <= p_j. */
static int64_t query_pos(const ref_cache* c, int b, int T, int j)
{
    return (int64_t)c->seq_lens[b] - T + j;
}

/* Full mode ([TLDR] paragraph 3): score every visible position, keep a pool of
 * the min(pool_k, p+1) best (pool_k <= 16,384) and, from the same scores, the
 * min(top_k, p+1) best as this layer's attention set.  scores_out (nullable)
 * receives the p+1 fp64 scores. */
int ref_index_full(const ref_cache* c, int b, int T, int j, int q_dtype, const void* q, const float* w,
                   int H_I, int pool_k, int top_k, int32_t* pool_idx, int32_t* topk_idx, double* scores_out)
{
    if (top_k > pool_k || pool_k > 16384 || top_k < 0) return REF_ERR_ARG;
    int64_t p = query_pos(c, b, T, j);
    if (p < 0) return REF_ERR_ARG;
    int64_t n = p + 1;
    double* s = scores_out ? scores_out : (double*)malloc(sizeof(double) * (size_t)n);
    if (!s) return REF_ERR_ARG;
    int rc = ref_index_scores(c, b, n, NULL, q_dtype, q, H_I, w, s);
    if (!rc) rc = ref_select_top(s, NULL, n, pool_k, pool_idx);
    if (!rc) rc = ref_select_top(s, NULL, n, top_k, topk_idx);
    if (!scores_out) free(s);
    return rc;
}

/* Reindex mode ([TLDR] paragraph 3, "rescore a shared candidate set"): score
 * only the valid (non-negative) pool entries with this layer's own query and
 * head weights, keep the min(top_k, |pool|) best.  scores_out (nullable)
 * receives one fp64 score per pool entry (NaN for padding). */
int ref_index_reindex(const ref_cache* c, int b, int T, int j, int q_dtype, const void* q, const float* w,
                      int H_I, const int32_t* pool_idx, int pool_k, int top_k, int32_t* topk_idx,
                      double* scores_out)
{
    if (top_k > pool_k || pool_k > 16384 || top_k < 0) return REF_ERR_ARG;
    int64_t p = query_pos(c, b, T, j);
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)(pool_k > 0 ? pool_k : 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(pool_k > 0 ? pool_k : 1));
    if (!pos || !s) { free(pos); free(s); return REF_ERR_ARG; }
    int64_t n = 0;
    int rc = REF_OK;
    for (int i = 0; i < pool_k; ++i) {
        if (scores_out) scores_out[i] = NAN;
        if (pool_idx[i] < 0) continue;
        if (pool_idx[i] > p) { rc = REF_ERR_BOUNDS; break; }
        pos[n++] = pool_idx[i];
    }
    if (!rc) rc = ref_index_scores(c, b, n, pos, q_dtype, q, H_I, w, s);
    if (!rc) rc = ref_select_top(s, pos, n, top_k, topk_idx);
    if (!rc && scores_out) {
        int64_t m = 0;
        for (int i = 0; i < pool_k; ++i)
            if (pool_idx[i] >= 0) scores_out[i] = s[m++];
    }
    free(pos);
    free(s);
    return rc;
}

/* Append-time pool maintenance for an in-flight request (the candidate     */
/* pool of [TLDR] paragraph 3 kept current as tokens are appended): the new  */
/* pool is the min(pool_k, |candidates|) best of the previous pool's valid   */
/* entries and the new positions t_new0 .. p, all scored with this query;   */
/* topk_idx receives the top_k best of the same candidates.  Previous pool   */
/* entries at or beyond t_new0 (or beyond p) are an argument error.          */
int ref_index_pool_update(const ref_cache* c, int b, int T, int j, int q_dtype, const void* q, const float* w,
                          int H_I, const int32_t* pool_prev, int pool_k, int64_t t_new0, int top_k,
                          int32_t* pool_idx, int32_t* topk_idx)
{
    if (top_k > pool_k || pool_k > 16384 || top_k < 0 || t_new0 < 0) return REF_ERR_ARG;
    int64_t p = query_pos(c, b, T, j);
    if (p < 0) return REF_ERR_ARG;
    int64_t n_new = p + 1 > t_new0 ? p + 1 - t_new0 : 0;
    int64_t cap = pool_k + n_new;
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
    if (!pos || !s) { free(pos); free(s); return REF_ERR_ARG; }
    int64_t n = 0;
    int rc = REF_OK;
    for (int i = 0; i < pool_k; ++i) {
        if (pool_prev[i] < 0) continue;
        if (pool_prev[i] >= t_new0 || pool_prev[i] > p) { rc = REF_ERR_ARG; break; }
        pos[n++] = pool_prev[i];
    }
    for (int64_t t = t_new0; t <= p && !rc; ++t) pos[n++] = (int32_t)t;
    if (!rc) rc = ref_index_scores(c, b, n, pos, q_dtype, q, H_I, w, s);
    if (!rc) rc = ref_select_top(s, pos, n, pool_k, pool_idx);
    if (!rc) rc = ref_select_top(s, pos, n, top_k, topk_idx);
    free(pos);
    free(s);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Sparse + sliding-window attention ([HN] key point 2, [TLDR] paragraphs 2  */
/* and 3).  S = window ∪ top-k without double counting, window =             */
/* [max(0, p-W+1), p]; -1 entries and entries beyond p are not visible.      */
/* For every head h, with v_t the dequantised latent of position t (key and  */
/* value at once):                                                           */
/*     z_t = sm_scale * q_h . v_t,  out_h = sum_{t in S} softmax(z)_t v_t,   */
/*     lse_h = log sum_{t in S} exp(z_t)                                     */
/* q is bf16 [H][D]; out is [H][D]; lse is [H] (nullable).                   */
/* ------------------------------------------------------------------------ */
/* The window rows come from `ring` when it is given (layer-local window      */
/* state, see ref_sparse_swa_attn_local), else from the FP4 cache.           */
static int sparse_swa_attn_rows(const ref_cache* c, const uint16_t* ring, int64_t ring_len, int b, int T, int j,
                                int H, const uint16_t* q, const int32_t* topk_idx, int top_k, int window,
                                double sm_scale, double* out, double* lse)
{
    int D = c->dim;
    int64_t p = query_pos(c, b, T, j);
    int64_t L = c->seq_lens[b];
    if (p < 0 || window < 0) return REF_ERR_ARG;
    if (sm_scale <= 0.0) sm_scale = 1.0 / sqrt((double)D);
    /* membership over positions 0..p: the union without double counting */
    unsigned char* in_s = (unsigned char*)calloc((size_t)(p + 1), 1);
    if (!in_s) return REF_ERR_ARG;
    int64_t lo = p - window + 1;
    if (lo < 0) lo = 0;
    for (int64_t t = lo; t <= p && window > 0; ++t) in_s[t] = 1;
    for (int i = 0; i < top_k; ++i) {
        int64_t t = topk_idx[i];
        if (t < -1 || t >= L) { free(in_s); return REF_ERR_BOUNDS; }
        if (t >= 0 && t <= p) in_s[t] = 1;
    }
    int64_t nS = 0;
    for (int64_t t = 0; t <= p; ++t) nS += in_s[t];
    int64_t* S = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nS > 0 ? nS : 1));
    double* v = (double*)malloc(sizeof(double) * (size_t)(nS > 0 ? nS : 1) * D);
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);
    double* z = (double*)malloc(sizeof(double) * (size_t)(nS > 0 ? nS : 1));
    if (!S || !v || !qd || !z) { free(in_s); free(S); free(v); free(qd); free(z); return REF_ERR_ARG; }
    int64_t k = 0;
    int rc = REF_OK;
    for (int64_t t = 0; t <= p; ++t) {
        if (!in_s[t]) continue;
        S[k] = t;
        if (ring && window > 0 && t >= lo) {
            /* a window position: its layer-local bf16 row, ring slot t mod ring_len */
            const uint16_t* r = ring + ((int64_t)b * ring_len + t % ring_len) * D;
            for (int d = 0; d < D; ++d) v[k * D + d] = (double)bf16_to_f32(r[d]);
        } else {
            int64_t slot = ref_slot(c, b, t);
            if (slot < 0) { rc = REF_ERR_BOUNDS; break; }
            ref_dequant_row(c->rows + slot * c->row_stride, D, v + k * D);
        }
        ++k;
    }
    for (int h = 0; h < H && !rc; ++h) {
        for (int d = 0; d < D; ++d) qd[d] = (double)bf16_to_f32(q[(int64_t)h * D + d]);
        if (nS == 0) {
            for (int d = 0; d < D; ++d) out[(int64_t)h * D + d] = 0.0;
            if (lse) lse[h] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int64_t i = 0; i < nS; ++i) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += qd[d] * v[i * D + d];
            z[i] = sm_scale * dot;
            if (z[i] > m) m = z[i];
        }
        double l = 0.0;
        for (int64_t i = 0; i < nS; ++i) { z[i] = exp(z[i] - m); l += z[i]; }
        for (int d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t i = 0; i < nS; ++i) acc += z[i] * v[i * D + d];
            out[(int64_t)h * D + d] = acc / l;
        }
        if (lse) lse[h] = m + log(l);
    }
    free(in_s); free(S); free(v); free(qd); free(z);
    return rc;
}

int ref_sparse_swa_attn(const ref_cache* c, int b, int T, int j, int H, const uint16_t* q,
                        const int32_t* topk_idx, int top_k, int window, double sm_scale,
                        double* out, double* lse)
{
    return sparse_swa_attn_rows(c, NULL, 0, b, T, j, H, q, topk_idx, top_k, window, sm_scale, out, lse);
}

/* ------------------------------------------------------------------------ */
/* Sparse attention with layer-local window state ([FANOUT] item 2: the      */
/* modes share global KV and sparse selections while queries and the        */
/* sliding-window state stay layer-local; [TLDR] paragraph 2: the window     */
/* runs in every layer and its states are rebuilt from the last 128          */
/* tokens).  The attended set S is the one of ref_sparse_swa_attn; a         */
/* position of the window takes its row from this layer's bf16 ring          */
/* [batch][ring_len][D] (position t at slot t mod ring_len, ring_len >=      */
/* window), every other position its dequantised FP4 row from the shared     */
/* cache.                                                                    */
/* ------------------------------------------------------------------------ */
int ref_sparse_swa_attn_local(const ref_cache* c, const uint16_t* ring, int64_t ring_len, int b, int T, int j,
                              int H, const uint16_t* q, const int32_t* topk_idx, int top_k, int window,
                              double sm_scale, double* out, double* lse)
{
    if (!ring || ring_len < window || ring_len < 1) return REF_ERR_ARG;
    return sparse_swa_attn_rows(c, ring, ring_len, b, T, j, H, q, topk_idx, top_k, window, sm_scale, out, lse);
}

/* ------------------------------------------------------------------------ */
/* Merge of attention partials over disjoint parts of one attended set (a    */
/* context sharded over devices, each attending over its own part): with     */
/* part i's output O_i and log-sum-exp l_i per head,                         */
/*     l = log sum_i exp(l_i),   O = sum_i exp(l_i - l) O_i.                 */
/* A part with l_i = -inf (nothing attended) contributes nothing; if every   */
/* part is empty the result is O = 0, l = -inf.                              */
/* outs is [n_parts][H][D], lses is [n_parts][H].                            */
/* ------------------------------------------------------------------------ */
int ref_lse_merge(int n_parts, int H, int D, const double* outs, const double* lses, double* out, double* lse)
{
    if (n_parts < 1 || H < 1 || D < 1) return REF_ERR_ARG;
    for (int h = 0; h < H; ++h) {
        double m = -INFINITY;
        for (int i = 0; i < n_parts; ++i)
            if (lses[(int64_t)i * H + h] > m) m = lses[(int64_t)i * H + h];
        for (int d = 0; d < D; ++d) out[(int64_t)h * D + d] = 0.0;
        if (m == -INFINITY) {
            lse[h] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int i = 0; i < n_parts; ++i) sum += exp(lses[(int64_t)i * H + h] - m);
        double l = m + log(sum);
        for (int i = 0; i < n_parts; ++i) {
            double wgt = exp(lses[(int64_t)i * H + h] - l);
            for (int d = 0; d < D; ++d) out[(int64_t)h * D + d] += wgt * outs[((int64_t)i * H + h) * D + d];
        }
        lse[h] = l;
    }
    return REF_OK;
}

/* ------------------------------------------------------------------------ */
/* Brute-force dense attention over every visible position 0..p, written     */
/* separately from the sparse routine (two passes over the cache, no set     */
/* construction).  When top-k covers the whole visible context the sparse    */
/* routine must agree with it.                                               */
/* ------------------------------------------------------------------------ */
int ref_dense_attn(const ref_cache* c, int b, int T, int j, int H, const uint16_t* q, double sm_scale,
                   double* out, double* lse)
{
    int D = c->dim;
    int64_t p = query_pos(c, b, T, j);
    if (p < 0) return REF_ERR_ARG;
    if (sm_scale <= 0.0) sm_scale = 1.0 / sqrt((double)D);
    double* row = (double*)malloc(sizeof(double) * (size_t)D);
    if (!row) return REF_ERR_ARG;
    for (int h = 0; h < H; ++h) {
        const uint16_t* qh = q + (int64_t)h * D;
        /* pass 1: the largest logit */
        double m = -INFINITY;
        for (int64_t t = 0; t <= p; ++t) {
            int64_t slot = ref_slot(c, b, t);
            if (slot < 0) { free(row); return REF_ERR_BOUNDS; }
            ref_dequant_row(c->rows + slot * c->row_stride, D, row);
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += (double)bf16_to_f32(qh[d]) * row[d];
            if (sm_scale * dot > m) m = sm_scale * dot;
        }
        /* pass 2: weights and weighted sum */
        double denom = 0.0;
        for (int d = 0; d < D; ++d) out[(int64_t)h * D + d] = 0.0;
        for (int64_t t = 0; t <= p; ++t) {
            int64_t slot = ref_slot(c, b, t);
            ref_dequant_row(c->rows + slot * c->row_stride, D, row);
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += (double)bf16_to_f32(qh[d]) * row[d];
            double e = exp(sm_scale * dot - m);
            denom += e;
            for (int d = 0; d < D; ++d) out[(int64_t)h * D + d] += e * row[d];
        }
        for (int d = 0; d < D; ++d) out[(int64_t)h * D + d] /= denom;
        if (lse) lse[h] = m + log(denom);
    }
    free(row);
    return REF_OK;
}
