/*
 * Lightning Indexer forward pass (and, at the end of the file, its backward with the KL loss):
 * plain CPU oracle.
 *
 * TEST INFRASTRUCTURE. This file is the slow, obviously correct reference that the CUDA library
 * is checked against. Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg may load it. It shares no code, header, table or helper with the CUDA library, and the
 * library never calls it.
 *
 * What it computes, step by step, in the order the pages give it:
 *
 *   1. Per batch b, the query length L1_b and key length L2_b (lightning_indexer, "Constraints":
 *      cu_seqlens are cumulative token counts, seqused_* are valid-token counts per batch;
 *      aclnnLightningIndexerV2, constraints: TND padding of query rows past seqused_q, and
 *      seqused_k being required for the paged key layout).
 *   2. The key window of query row i (custom_pypto.npu_lightning_indexer_pto, sparse_mode:
 *      0 = no mask, 3 = right-down causal, i.e. the lower triangle anchored at the bottom-right
 *      corner): mode 0 keeps 0 <= j < L2_b, mode 3 additionally keeps j <= i + L2_b - L1_b.
 *      Compressed keys (lightning_indexer, "Prototype": cmp_ratio and cmp_residual_k;
 *      "Constraints": cmp_residual_k[b] < cmp_ratio, required with cmp_ratio > 1 and mask 3):
 *      [reading] key j of batch b stands for original tokens [j*r, (j+1)*r) of a sequence of
 *      L2_b*r + cmp_residual_k[b] tokens, and under mode 3 it is kept when its last token is
 *      visible: (j+1)*r - 1 <= i + L2_b*r + cmp_residual_k[b] - L1_b. The pages state no rule
 *      and give no worked values for it: parity of this reading is unpinned beyond the
 *      whole-block relation the pins check.
 *   3. The index score (custom_pypto.npu_lightning_indexer_pto, formula in the function
 *      description; lightning_indexer, "Function" steps 1-3 and "Formula"):
 *         I[i,j] = sum_h w[i,h] * ReLU( q[i,h,:] . k[j,:] )
 *      with no 1/sqrt(d) scale (the scale belongs only to the main attention softmax in
 *      torch_npu.npu_sparse_lightning_indexer_grad_kl_loss, formula 2).
 *   4. Top-k selection per row, output sorted (npu_sparse_lightning_indexer_grad_kl_loss,
 *      parameter sparse_indices: "sorted" token indices), padded with index -1 and value -inf
 *      (aclnnLightningIndexerV2 and lightning_indexer, constraints), indices shifted by
 *      output_idx_offset (aclnnLightningIndexerV2 constraints: the shifted index must not exceed
 *      INT32_MAX).
 *   5. Merge of key-range shards (the split-merge step that follows a key-range split of one
 *      row): [reading] the pages select over the whole window of a row, so the top-k of a row
 *      whose keys were split into disjoint ranges, each range selected on its own with its
 *      keys' global indices, is the top-k of the union of the per-range lists under the same
 *      order. orc_merge_topk writes out exactly that: all valid entries of all lists, one sort,
 *      the first topk kept.
 *
 * Precision. q and k arrive as bf16 or fp16 bit patterns (lightning_indexer, "Constraints": q
 * and k share one type; the single-operator example passes fp16 q and k with fp32 w), or as fp8
 * e4m3 codes with q_descale and k_descale (aclnnLightningIndexerV2, parameter dimensions: the
 * pages name these two arguments and nothing more; [reading] dequantized q = code x
 * q_descale[row, head], k = code x k_descale[key]; parity of this reading is unpinned beyond the
 * fp8 decoding and the scaling laws the pins check). w arrives as bf16, fp16 or fp32; every
 * product and sum is taken in fp64, so the score is the exact real value up to fp64 rounding. The selection decision is then taken on
 * the score rounded once to fp32, the precision the CUDA kernels decide in, and -0 is treated as
 * +0. Order: score descending, then key index ascending (the pages only say "deterministic").
 *
 * Every point the pages leave open is taken with the plainest reading the rest of the pages
 * support, and each such reading is marked [reading] below where it is applied.
 *
 * Planted mistakes. Building with -DORC_MUTANT=n plants mistake n (see the ORC_MUTANT blocks).
 * A test builds each mutant and checks that the pins catch it. A normal build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

enum { ORC_BSND = 0, ORC_TND = 1, ORC_PA_BSND = 2 };
enum { ORC_BF16 = 0, ORC_FP16 = 1, ORC_FP32 = 2, ORC_FP8_E4M3 = 3 };
enum { ORC_OK = 0, ORC_EARG = 1, ORC_EDATA = 2, ORC_ENOMEM = 3 };

/* One problem. All arrays are host memory in the layouts the pages give:
 *   q: BSND (B, S1, N1, D) or TND (T1, N1, D)
 *   k: BSND (B, S2, 1, D), TND (T2, 1, D) or PA_BSND (num_blocks, block_size, 1, D)
 *   w: (B, S1, N1) or (T1, N1)
 * Optional arrays are NULL when absent. */
typedef struct {
    const void *q, *k;              /* bf16 / fp16 bit patterns (2 bytes) or fp8 e4m3 (1 byte)  */
    const void *w;                  /* bf16 or fp16 bit patterns, or fp32 values (dtype_w)      */
    const int32_t *cu_seqlens_q, *cu_seqlens_k;
    const int32_t *seqused_q, *seqused_k;
    const int32_t *block_table;
    const int32_t *output_idx_offset;
    int64_t block_table_stride;
    int32_t batch;
    int32_t q_len;      /* BSND: S1; TND: T1 */
    int32_t k_len;      /* BSND: S2; TND: T2; PA_BSND: unused */
    int32_t num_blocks, block_size;
    int32_t n_heads, head_dim, topk;
    int32_t layout_q, layout_k, mask_mode;
    const int32_t *cmp_residual_k;  /* [B] or NULL: tokens past the last whole compressed key */
    int32_t cmp_ratio;              /* original tokens per key; 0 or 1 = keys not compressed  */
    int32_t dtype_qk, dtype_w;      /* ORC_BF16 / ORC_FP16 / ORC_FP8_E4M3 (q, k); ORC_BF16 /
                                       ORC_FP16 / ORC_FP32 (w)                                  */
    const float *q_descale;         /* fp8 q, k: [rows * N1] (laid out like w) and one value  */
    const float *k_descale;         /* per key row (laid out like k without D); NULL otherwise */
} orc_problem;

static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16: sign, 5 exponent bits (bias 15), 10 fraction bits. */
static double fp16_value(uint16_t bits)
{
    const int sign = bits >> 15, e = (bits >> 10) & 0x1f, f = bits & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                        /* subnormal: f * 2^-24        */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
#if ORC_MUTANT == 13
        v = ldexp(1024.0 + f, e - 24);                    /* mistake: exponent bias 14   */
#else
        v = ldexp(1024.0 + f, e - 25);                    /* (1 + f/1024) * 2^(e - 15)   */
#endif
    return sign ? -v : v;
}

/* OCP 8-bit float E4M3 (the "fn" variant: no infinities): sign, 4 exponent bits (bias 7),
 * 3 fraction bits; exponent 15 with fraction 7 is NaN, so the largest value is 448. */
static double fp8_e4m3_value(uint8_t bits)
{
    const int sign = bits >> 7, e = (bits >> 3) & 0xf, f = bits & 0x7;
    double v;
    if (e == 0)
        v = ldexp((double)f, -9);                         /* subnormal: (f/8) * 2^-6     */
    else if (e == 15 && f == 7)
        v = NAN;
    else
        v = ldexp(8.0 + f, e - 10);                       /* (1 + f/8) * 2^(e - 7)       */
    return sign ? -v : v;
}

/* Element i of q or k (a 2-byte or 1-byte array by dtype_qk) as a real number. */
static double qk_value(const orc_problem *p, const void *arr, int64_t i)
{
    if (p->dtype_qk == ORC_FP8_E4M3) return fp8_e4m3_value(((const uint8_t *)arr)[i]);
    const uint16_t bits = ((const uint16_t *)arr)[i];
    return p->dtype_qk == ORC_FP16 ? fp16_value(bits) : bf16_value(bits);
}

static double w_value(const orc_problem *p, int64_t idx)
{
    if (p->dtype_w == ORC_FP32) {
        float f;
        memcpy(&f, (const char *)p->w + 4 * idx, sizeof f);
        return (double)f;
    }
    const uint16_t bits = ((const uint16_t *)p->w)[idx];
    return p->dtype_w == ORC_FP16 ? fp16_value(bits) : bf16_value(bits);
}

static int64_t orc_num_rows(const orc_problem *p)
{
    return p->layout_q == ORC_TND ? (int64_t)p->q_len : (int64_t)p->batch * p->q_len;
}

/* Step 1: which batch a query row belongs to, its position there, and the lengths. */
typedef struct {
    int32_t b, i;          /* batch and row position within the batch                      */
    int64_t L1, L2;        /* query rows allocated / keys valid for the batch              */
    int64_t L1_used;       /* query rows in use (seqused_q), used for validity + alignment */
    int64_t res;           /* compressed keys: residual original tokens of the batch           */
} orc_row;

static int orc_locate(const orc_problem *p, int64_t r, orc_row *o)
{
    if (p->layout_q == ORC_TND) {
        int b = -1;
        for (int bb = 0; bb < p->batch; ++bb)
            if (p->cu_seqlens_q[bb] <= r && r < p->cu_seqlens_q[bb + 1]) { b = bb; break; }
        if (b < 0) {            /* row not covered by any batch: no valid keys */
            o->b = -1; o->i = 0; o->L1 = 0; o->L2 = 0; o->L1_used = 0; o->res = 0;
            return ORC_OK;
        }
        o->b = b;
        o->i = (int32_t)(r - p->cu_seqlens_q[b]);
        o->L1 = p->cu_seqlens_q[b + 1] - p->cu_seqlens_q[b];
    } else {
        o->b = (int32_t)(r / p->q_len);
        o->i = (int32_t)(r % p->q_len);
        o->L1 = p->q_len;
    }
    if (p->layout_k == ORC_TND)
        o->L2 = p->cu_seqlens_k[o->b + 1] - p->cu_seqlens_k[o->b];
    else if (p->layout_k == ORC_PA_BSND)
        o->L2 = p->seqused_k[o->b];
    else
        o->L2 = p->k_len;
    /* [reading] seqused_k, when given for a non-paged layout, is the valid key count. */
    if (p->seqused_k && p->layout_k != ORC_PA_BSND && p->seqused_k[o->b] < o->L2)
        o->L2 = p->seqused_k[o->b];
    o->L1_used = o->L1;
    if (p->seqused_q && p->seqused_q[o->b] < o->L1_used)
        o->L1_used = p->seqused_q[o->b];
    o->res = p->cmp_residual_k ? p->cmp_residual_k[o->b] : 0;
    return ORC_OK;
}

/* Step 2: the window is always a prefix [0, hi) of the batch's keys. */
static int64_t orc_window(const orc_problem *p, const orc_row *o)
{
    if (o->b < 0 || o->i >= o->L1_used || o->L2 <= 0) return 0;
    int64_t hi = o->L2;
    if (p->mask_mode == 3 && p->cmp_ratio > 1) {
        /* compressed keys: count keys from the first while each one's last original token is
           visible to row i (original tokens aligned right-down like uncompressed keys) */
        const int64_t r = p->cmp_ratio;
        const int64_t horizon = (int64_t)o->i + o->L2 * r + o->res - o->L1_used;
        int64_t n = 0;
#if ORC_MUTANT == 12
        while (n < o->L2 && n * r <= horizon) ++n;           /* mistake: first token visible */
#else
        while (n < o->L2 && (n + 1) * r - 1 <= horizon) ++n;
#endif
        return n;
    }
    if (p->mask_mode == 3) {
        /* [reading] right-down causal aligns the last used query row with the last key. */
#if ORC_MUTANT == 3
        int64_t lim = o->i + 1;                       /* mistake: top-left alignment */
#else
        int64_t lim = (int64_t)o->i + o->L2 - o->L1_used + 1;
#endif
        if (lim < hi) hi = lim;
    }
    return hi < 0 ? 0 : hi;
}

/* Row of k (in units of D elements) holding key j of batch b (logical position within the
 * batch's key sequence). */
static int64_t orc_key_row(const orc_problem *p, int32_t b, int64_t j)
{
    if (p->layout_k == ORC_TND) {
#if ORC_MUTANT == 8
        return (int64_t)p->cu_seqlens_q[b] + j;   /* mistake: query offsets */
#else
        return (int64_t)p->cu_seqlens_k[b] + j;
#endif
    }
    if (p->layout_k == ORC_PA_BSND) {
#if ORC_MUTANT == 7
        (void)b;
        return j;                                 /* mistake: block table ignored */
#else
        int64_t blk = p->block_table[(int64_t)b * p->block_table_stride + j / p->block_size];
        return blk * p->block_size + j % p->block_size;
#endif
    }
    return (int64_t)b * p->k_len + j;
}

/* Row of q (in units of D elements) holding head h of query row r. */
static int64_t orc_query_row(const orc_problem *p, int64_t r, int32_t h)
{
#if ORC_MUTANT == 6
    return (int64_t)h * orc_num_rows(p) + r;      /* mistake: head and row strides exchanged */
#else
    return r * p->n_heads + h;
#endif
}

/* Step 3: the exact score of row r against key j, in fp64. */
static double orc_score(const orc_problem *p, int64_t r, const orc_row *o, int64_t j)
{
    const int64_t D = p->head_dim;
    const int64_t kr = orc_key_row(p, o->b, j);
    double I = 0.0;
#if ORC_MUTANT == 1
    double sum_ws = 0.0;
#endif
    for (int32_t h = 0; h < p->n_heads; ++h) {
        const int64_t qr = orc_query_row(p, r, h);
        double s = 0.0;
        for (int32_t d = 0; d < p->head_dim; ++d)
            s += qk_value(p, p->q, qr * D + d) * qk_value(p, p->k, kr * D + d);
        /* [reading] fp8 q and k are quantized values: q_descale[r, h] and k_descale[key row]
         * scale them back (the pages name q_descale and k_descale and their dimensions only) */
        if (p->dtype_qk == ORC_FP8_E4M3)
#if ORC_MUTANT == 15
            s *= (double)p->q_descale[r * p->n_heads + h];    /* mistake: k_descale dropped */
#else
            s *= (double)p->q_descale[r * p->n_heads + h] * (double)p->k_descale[kr];
#endif
        double wh = w_value(p, r * p->n_heads + h);
#if ORC_MUTANT == 1
        sum_ws += wh * s;                              /* mistake: ReLU after the head sum */
#elif ORC_MUTANT == 2
        (void)wh;
        I += (s > 0.0 ? s : 0.0);                      /* mistake: weights dropped */
#elif ORC_MUTANT == 9
        I += wh * s;                                   /* mistake: ReLU dropped */
#elif ORC_MUTANT == 5
        if (h == 0) I = wh * (s > 0.0 ? s : 0.0);     /* mistake: sum seeded with a -0 term */
        else I += wh * (s > 0.0 ? s : 0.0);
#else
        I += wh * (s > 0.0 ? s : 0.0);
#endif
    }
#if ORC_MUTANT == 1
    I = sum_ws > 0.0 ? sum_ws : 0.0;
#endif
    return I;
}

typedef struct { float v; int64_t j; } orc_entry;

/* Step 4 order: score descending, then key index ascending. */
static int orc_cmp(const void *a, const void *b)
{
    const orc_entry *x = (const orc_entry *)a, *y = (const orc_entry *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
#if ORC_MUTANT == 4
    return (x->j < y->j) ? 1 : (x->j > y->j) ? -1 : 0;  /* mistake: higher index first */
#else
    return (x->j < y->j) ? -1 : (x->j > y->j) ? 1 : 0;
#endif
}

static float orc_to_f32(double I)
{
    float v = (float)I;
#if ORC_MUTANT != 5
    if (v == 0.0f) v = 0.0f;   /* -0 counts as +0 */
#endif
    return v;
}

static int orc_check(const orc_problem *p)
{
    if (!p || !p->q || !p->k || !p->w) return ORC_EARG;
    if (p->n_heads < 1 || p->head_dim < 1 || p->topk < 1 || p->batch < 0) return ORC_EARG;
    if (p->mask_mode != 0 && p->mask_mode != 3) return ORC_EARG;
    if (p->layout_q != ORC_BSND && p->layout_q != ORC_TND) return ORC_EARG;
    if (p->layout_k < ORC_BSND || p->layout_k > ORC_PA_BSND) return ORC_EARG;
    if (p->layout_q == ORC_TND && !p->cu_seqlens_q) return ORC_EARG;
    if (p->layout_k == ORC_TND && !p->cu_seqlens_k) return ORC_EARG;
    if (p->layout_k == ORC_PA_BSND && (!p->seqused_k || !p->block_table || p->block_size < 1))
        return ORC_EARG;
    if (p->cmp_ratio < 0) return ORC_EARG;
    if (p->dtype_qk != ORC_BF16 && p->dtype_qk != ORC_FP16 && p->dtype_qk != ORC_FP8_E4M3)
        return ORC_EARG;
    if (p->dtype_qk == ORC_FP8_E4M3 && (!p->q_descale || !p->k_descale)) return ORC_EARG;
    if (p->dtype_w != ORC_BF16 && p->dtype_w != ORC_FP16 && p->dtype_w != ORC_FP32) return ORC_EARG;
    if (p->cmp_residual_k)
        for (int b = 0; b < p->batch; ++b)
            if (p->cmp_residual_k[b] < 0 || p->cmp_residual_k[b] >= (p->cmp_ratio > 1 ? p->cmp_ratio : 1))
                return ORC_EDATA;
    return ORC_OK;
}

/* Number of query rows of the problem (B*S1 for BSND, T1 for TND). */
int64_t orc_rows(const orc_problem *p) { return orc_num_rows(p); }

/* The exact scores of one row over its window: scores[j] for 0 <= j < *hi (fp64).
 * scores must hold at least the batch's key count. */
int orc_scores(const orc_problem *p, int64_t r, double *scores, int64_t *hi)
{
    int rc = orc_check(p);
    if (rc) return rc;
    if (r < 0 || r >= orc_num_rows(p)) return ORC_EARG;
    orc_row o;
    orc_locate(p, r, &o);
    *hi = orc_window(p, &o);
    for (int64_t j = 0; j < *hi; ++j) scores[j] = orc_score(p, r, &o, j);
    return ORC_OK;
}

/* The window length, batch and in-batch position of a row. */
int orc_row_info(const orc_problem *p, int64_t r, int64_t *hi, int32_t *b, int32_t *i)
{
    int rc = orc_check(p);
    if (rc) return rc;
    if (r < 0 || r >= orc_num_rows(p)) return ORC_EARG;
    orc_row o;
    orc_locate(p, r, &o);
    *hi = orc_window(p, &o);
    *b = o.b;
    *i = o.i;
    return ORC_OK;
}

/* The exact score of one (row, key) pair; ORC_EARG when j is outside the row's window. */
int orc_score_at(const orc_problem *p, int64_t r, int64_t j, double *out)
{
    int rc = orc_check(p);
    if (rc) return rc;
    if (r < 0 || r >= orc_num_rows(p)) return ORC_EARG;
    orc_row o;
    orc_locate(p, r, &o);
    if (j < 0 || j >= orc_window(p, &o)) return ORC_EARG;
    *out = orc_score(p, r, &o, j);
    return ORC_OK;
}

/* Top-k of the listed rows (all rows when rows == NULL). Row n of the output is the n-th listed
 * row: out_idx[n*topk + m], out_val[n*topk + m]. When row_maxabs is not NULL it receives, per
 * listed row, the largest |I| over the row's window (0 for an empty window). Returns ORC_EDATA
 * when an offset index would pass INT32_MAX. */
int orc_topk(const orc_problem *p, const int64_t *rows, int64_t n_rows,
             int32_t *out_idx, float *out_val, double *row_maxabs)
{
    int rc = orc_check(p);
    if (rc) return rc;
    const int64_t R = rows ? n_rows : orc_num_rows(p);
    int64_t cap = 0;
    for (int64_t n = 0; n < R; ++n) {
        int64_t r = rows ? rows[n] : n;
        if (r < 0 || r >= orc_num_rows(p)) return ORC_EARG;
        orc_row o;
        orc_locate(p, r, &o);
        int64_t hi = orc_window(p, &o);
        if (hi > cap) cap = hi;
    }
    orc_entry *e = (orc_entry *)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(orc_entry));
    if (!e) return ORC_ENOMEM;
    rc = ORC_OK;
    for (int64_t n = 0; n < R; ++n) {
        int64_t r = rows ? rows[n] : n;
        orc_row o;
        orc_locate(p, r, &o);
        int64_t hi = orc_window(p, &o);
        double maxabs = 0.0;
        for (int64_t j = 0; j < hi; ++j) {
            double I = orc_score(p, r, &o, j);
            if (fabs(I) > maxabs) maxabs = fabs(I);
            e[j].v = orc_to_f32(I);
            e[j].j = j;
        }
        if (row_maxabs) row_maxabs[n] = maxabs;
        qsort(e, (size_t)hi, sizeof(orc_entry), orc_cmp);
        int64_t m = hi < p->topk ? hi : p->topk;
        int64_t off = 0;
#if ORC_MUTANT != 10
        if (p->output_idx_offset && o.b >= 0) off = p->output_idx_offset[o.b];
#endif
        for (int64_t s = 0; s < p->topk; ++s) {
            int32_t *ix = out_idx + n * p->topk + s;
            float *vx = out_val + n * p->topk + s;
            if (s < m) {
                int64_t idx = e[s].j + off;
                if (idx > INT32_MAX) { rc = ORC_EDATA; idx = -1; }
                *ix = (int32_t)idx;
                *vx = e[s].v;
            } else {
#if ORC_MUTANT == 11
                *ix = 0;                                /* mistake: wrong padding */
                *vx = 0.0f;
#else
                *ix = -1;
                *vx = -INFINITY;
#endif
            }
        }
    }
    free(e);
    return rc;
}

/* Step 5: top-k of the union of n_lists per-row lists. List l, row r, entry e is
 * idx[(l*rows + r)*topk_in + e] / val[...]; an entry with a negative index is padding. Output row
 * r holds the first topk_out of all valid entries of row r in step 4's order (score descending,
 * index ascending), then -1 / -inf. The decision is taken on the fp32 values as given, -0 as
 * +0. Returns ORC_EARG for bad sizes. */
int orc_merge_topk(int64_t rows, int32_t n_lists, int32_t topk_in, const int32_t *idx,
                   const float *val, int32_t topk_out, int32_t *out_idx, float *out_val)
{
    if (rows < 0 || n_lists < 1 || topk_in < 1 || topk_out < 1 || !idx || !val || !out_idx ||
        !out_val)
        return ORC_EARG;
    int32_t lists = n_lists;
#if ORC_MUTANT == 14
    lists = n_lists - 1;                          /* mistake: the last list is dropped */
#endif
    orc_entry *e = (orc_entry *)malloc((size_t)lists * (size_t)topk_in * sizeof(orc_entry) + 1);
    if (!e) return ORC_ENOMEM;
    for (int64_t r = 0; r < rows; ++r) {
        int64_t n = 0;
        for (int32_t l = 0; l < lists; ++l) {
            for (int32_t k = 0; k < topk_in; ++k) {
                const int64_t at = ((int64_t)l * rows + r) * topk_in + k;
                if (idx[at] < 0) continue;
                e[n].v = val[at] == 0.0f ? 0.0f : val[at];
                e[n].j = idx[at];
                ++n;
            }
        }
        qsort(e, (size_t)n, sizeof(orc_entry), orc_cmp);
        for (int32_t s = 0; s < topk_out; ++s) {
            out_idx[r * topk_out + s] = s < n ? (int32_t)e[s].j : -1;
            out_val[r * topk_out + s] = s < n ? e[s].v : -INFINITY;
        }
    }
    free(e);
    return ORC_OK;
}

/* ---- Indexer backward with the KL loss ------------------------------------------------------
 *
 * torch_npu.npu_sparse_lightning_indexer_grad_kl_loss, "计算公式" 1-4. For query row r (batch b)
 * and its selected keys s (sparse_indices[r, :], positions inside batch b's keys, -1 = padding):
 *   1. I[s]   = sum_h w[r,h] ReLU(qi[r,h,:] . ki[s,:])                   (the indexer score)
 *   2. P_g[s] = exp(scale (q[r,g,:] . k[s,:] + q_rope[r,g,:] . k_rope[s,:]) - max[r,g]) / sum[r,g]
 *      (the main attention softmax, rebuilt from its forward statistics softmax_max/_sum)
 *   3. p[s]   = sum_g P_g[s] / sum_{s'} sum_g P_g[s']   [reading] the head sum of the main
 *      attention scores normalised to 1 over the selected keys ("L1 normalisation along the
 *      context direction"); loss_r = sum_s p[s] log(p[s] / softmax(I)[s]) with 0 log 0 = 0, and
 *      the loss returned is the sum over rows [reading: the formula's sum over t].
 *   4. dI[s] = softmax(I)[s] - p[s];  dw[r,h] = sum_s dI[s] ReLU(S[h,s]) with S = qi . ki;
 *      dS[h,s] = dI[s] w[r,h] [S[h,s] > 0];  dqi[r,h,:] = sum_s dS[h,s] ki[s,:];
 *      dki[s,:] += sum_h dS[h,s] qi[r,h,:]  (summed over every row that selected key s).
 * Inputs are real values (the wrapper decodes bf16/fp16 exactly); everything is fp64. Rows with
 * no selected key add nothing. */
typedef struct {
    const double *q, *k;            /* main attention: q [rows, G, Dm], k [key rows, Dm]        */
    const double *q_rope, *k_rope;  /* [rows, G, Dr] / [key rows, Dr], or NULL when Dr == 0    */
    const double *qi, *ki, *w;      /* indexer: qi [rows, H, Di], ki [key rows, Di], w [rows, H]*/
    const int32_t *sparse_indices;  /* [rows, topk]                                            */
    const int64_t *key_base;        /* [rows]: key row of position 0 of the row's batch        */
    const double *softmax_max, *softmax_sum;   /* [rows, G]                                    */
    double scale;
    int64_t rows, key_rows;
    int32_t G, Dm, Dr, H, Di, topk;
} orc_kl;

static double dot(const double *a, const double *b, int32_t n)
{
    double s = 0.0;
    for (int32_t d = 0; d < n; ++d) s += a[d] * b[d];
    return s;
}

/* loss (scalar), d_qi [rows, H, Di], d_ki [key rows, Di], d_w [rows, H]; the gradient arrays are
 * overwritten. Returns ORC_EARG for bad sizes, ORC_EDATA for a selected key outside the keys. */
int orc_kl_grad(const orc_kl *a, double *loss, double *d_qi, double *d_ki, double *d_w)
{
    if (!a || !loss || !d_qi || !d_ki || !d_w || a->rows < 0 || a->G < 1 || a->Dm < 1 ||
        a->Dr < 0 || a->H < 1 || a->Di < 1 || a->topk < 1 || (a->Dr > 0 && (!a->q_rope || !a->k_rope)))
        return ORC_EARG;
    const int32_t K = a->topk, H = a->H, G = a->G, Di = a->Di;
    memset(d_qi, 0, sizeof(double) * (size_t)a->rows * H * Di);
    memset(d_ki, 0, sizeof(double) * (size_t)a->key_rows * Di);
    memset(d_w, 0, sizeof(double) * (size_t)a->rows * H);
    double *I = (double *)malloc(sizeof(double) * K), *p = (double *)malloc(sizeof(double) * K);
    double *sig = (double *)malloc(sizeof(double) * K), *S = (double *)malloc(sizeof(double) * K * H);
    int64_t *kr = (int64_t *)malloc(sizeof(int64_t) * K);
    if (!I || !p || !sig || !S || !kr) {
        free(I); free(p); free(sig); free(S); free(kr);
        return ORC_ENOMEM;
    }
    double total = 0.0;
    int rc = ORC_OK;
    for (int64_t r = 0; r < a->rows && rc == ORC_OK; ++r) {
        int32_t n = 0;
        for (int32_t e = 0; e < K; ++e) {
            const int32_t j = a->sparse_indices[r * K + e];
            if (j < 0) continue;
            const int64_t row = a->key_base[r] + j;
            if (row >= a->key_rows) { rc = ORC_EDATA; break; }
            kr[n++] = row;
        }
        if (rc != ORC_OK || n == 0) continue;
        /* 1. indexer scores */
        for (int32_t s = 0; s < n; ++s) {
            I[s] = 0.0;
            for (int32_t h = 0; h < H; ++h) {
                const double v = dot(a->qi + (r * H + h) * Di, a->ki + kr[s] * Di, Di);
                S[s * H + h] = v;
                I[s] += a->w[r * H + h] * (v > 0.0 ? v : 0.0);
            }
        }
        /* 2-3. target distribution from the main attention */
        double psum = 0.0;
        for (int32_t s = 0; s < n; ++s) {
            p[s] = 0.0;
            for (int32_t g = 0; g < G; ++g) {
                double x = dot(a->q + (r * G + g) * a->Dm, a->k + kr[s] * a->Dm, a->Dm);
                if (a->Dr > 0) x += dot(a->q_rope + (r * G + g) * a->Dr, a->k_rope + kr[s] * a->Dr, a->Dr);
                p[s] += exp(a->scale * x - a->softmax_max[r * G + g]) / a->softmax_sum[r * G + g];
            }
            psum += p[s];
        }
#if ORC_MUTANT != 17
        for (int32_t s = 0; s < n; ++s) p[s] /= psum;          /* mutant 17 skips the L1 norm */
#else
        (void)psum;
#endif
        /* softmax of the indexer scores */
        double imax = I[0], ssum = 0.0;
        for (int32_t s = 1; s < n; ++s) imax = I[s] > imax ? I[s] : imax;
        for (int32_t s = 0; s < n; ++s) ssum += exp(I[s] - imax);
        for (int32_t s = 0; s < n; ++s) sig[s] = exp(I[s] - imax) / ssum;
        for (int32_t s = 0; s < n; ++s)
            if (p[s] > 0.0) total += p[s] * (log(p[s]) - log(sig[s]));
        /* 4. gradients */
        for (int32_t s = 0; s < n; ++s) {
#if ORC_MUTANT == 16
            const double dI = p[s] - sig[s];                    /* mistake: sign of dI */
#else
            const double dI = sig[s] - p[s];
#endif
            for (int32_t h = 0; h < H; ++h) {
                const double v = S[s * H + h];
                if (v <= 0.0) continue;
                d_w[r * H + h] += dI * v;
                const double dS = dI * a->w[r * H + h];
                for (int32_t d = 0; d < Di; ++d) {
                    d_qi[(r * H + h) * Di + d] += dS * a->ki[kr[s] * Di + d];
                    d_ki[kr[s] * Di + d] += dS * a->qi[(r * H + h) * Di + d];
                }
            }
        }
    }
    free(I); free(p); free(sig); free(S); free(kr);
    *loss = total;
    return rc;
}

/* ---- Sparse attention over the selected keys ---------------------------------------------------
 *
 * The consumer of the indexer's output (aclnnLightningIndexerV2, "主要计算过程" step 3: the
 * selected indices are the attention's input; aclnnSparseFlashAttentionGrad, "Calculation formula":
 * the selected keys and values are gathered by the top-k indices, and only value = key is
 * supported). For query row r, head g and the row's selected keys s:
 *     x[s]  = scale (q[r,g,:] . k[s,:] + q_rope[r,g,:] . k_rope[s,:])
 *     m     = max_s x[s],   l = sum_s exp(x[s] - m)
 *     o[r,g,:] = sum_s exp(x[s] - m) / l * k[s,:]          [reading] the value rows are the key rows
 * and the forward statistics softmax_max = m, softmax_sum = l that the backward takes. A row with
 * no selected key gets o = 0, m = -inf, l = 0. fp64 from real-valued inputs. */
typedef struct {
    const double *q, *k, *q_rope, *k_rope;   /* q [rows, G, Dm], k [key rows, Dm], rope or NULL */
    const int32_t *sparse_indices;           /* [rows, topk], positions in the row's batch       */
    const int64_t *key_base;                 /* [rows]                                           */
    double scale;
    int64_t rows, key_rows;
    int32_t G, Dm, Dr, topk;
} orc_attn;

int orc_sparse_attention(const orc_attn *a, double *out, double *smax, double *ssum)
{
    if (!a || !out || !smax || !ssum || a->rows < 0 || a->G < 1 || a->Dm < 1 || a->Dr < 0 ||
        a->topk < 1 || (a->Dr > 0 && (!a->q_rope || !a->k_rope)))
        return ORC_EARG;
    const int32_t K = a->topk, G = a->G, Dm = a->Dm;
    double *x = (double *)malloc(sizeof(double) * K);
    int64_t *kr = (int64_t *)malloc(sizeof(int64_t) * K);
    if (!x || !kr) { free(x); free(kr); return ORC_ENOMEM; }
    int rc = ORC_OK;
    for (int64_t r = 0; r < a->rows && rc == ORC_OK; ++r) {
        int32_t n = 0;
        for (int32_t e = 0; e < K; ++e) {
            const int32_t j = a->sparse_indices[r * K + e];
            if (j < 0) continue;
            if (a->key_base[r] + j >= a->key_rows) { rc = ORC_EDATA; break; }
            kr[n++] = a->key_base[r] + j;
        }
        for (int32_t g = 0; g < G && rc == ORC_OK; ++g) {
            double *o = out + (r * G + g) * Dm;
            for (int32_t d = 0; d < Dm; ++d) o[d] = 0.0;
            if (n == 0) {
                smax[r * G + g] = -INFINITY;
                ssum[r * G + g] = 0.0;
                continue;
            }
            double m = -INFINITY, l = 0.0;
            for (int32_t s = 0; s < n; ++s) {
                x[s] = dot(a->q + (r * G + g) * Dm, a->k + kr[s] * Dm, Dm);
#if ORC_MUTANT != 18
                if (a->Dr > 0)
                    x[s] += dot(a->q_rope + (r * G + g) * a->Dr, a->k_rope + kr[s] * a->Dr, a->Dr);
#endif
                x[s] *= a->scale;
                if (x[s] > m) m = x[s];
            }
            for (int32_t s = 0; s < n; ++s) l += exp(x[s] - m);
            for (int32_t s = 0; s < n; ++s) {
                const double pw = exp(x[s] - m) / l;
                for (int32_t d = 0; d < Dm; ++d) o[d] += pw * a->k[kr[s] * Dm + d];
            }
            smax[r * G + g] = m;
            ssum[r * G + g] = l;
        }
    }
    free(x); free(kr);
    return rc;
}
