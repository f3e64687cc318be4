/*
 * fia_oracle.c -- CPU oracle for paged fused inference attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg call this file.  It shares no code, header or
 * constant with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (aclnnFusedInferAttentionScoreV4, "Formula"; V3 "Formula";
 * ATB PrefixEncoder parameter table):
 *
 *     out = Softmax(qkScale * Q K^T + bias) V
 *
 * one (sequence b, new token i, query head h) row at a time, in double
 * precision, with the paged K/V cache resolved naively through the block table
 * (paged attention: the blocks named by blockTables form one logically
 * contiguous K/V sequence -- V4 and V3 paged-attention bullets).
 *
 * Steps, per row:
 *   1. kvh = h / (headNum / kvHeadNum)               (GQA grouping, contiguous)
 *      qpos = kvSeqLen[b] - seqLen[b] + i            (new tokens are the last
 *                                                      seqLen[b] cache entries)
 *   2. for every logical kv position t < kvSeqLen[b]:
 *        blk = blockTables[b][t / blockSize], off = t % blockSize
 *        k_t = key[blk][off][kvh][:],  v_t = value[blk][off][kvh][:]   (BnBsH)
 *        k_t = key[blk][kvh][off][:],  v_t = value[blk][kvh][off][:]   (BnNBsD;
 *        V3 paged attention constraints: the cache is BnBsH or BnNBsD)
 *        int8 cache: k^ = kScale * (k + kOffset), v^ = vScale * (v + vOffset)
 *        per (kvh, d) channel (per-channel mode) or per (b, t) cached token
 *        (per-token mode, scale/offset [B, S], V3 fake-quantization
 *        bullets; K and V modes may differ); no offset given -> offset 0.
 *   3. causal (maskType 9, and 3 = ALiBi which includes causal): skip t > qpos
 *      band (V3 sparseMode 4): skip t < qpos - preTokens and t > qpos + nextTokens
 *   4. s_t = qkScale * sum_d q_d k_td
 *        + slope_h * (t - qpos)          (maskType 3)
 *        + pse[b][h][i][t]               (when a pse tensor is given)
 *   5. m = max_t s_t  (and the sink logit, when given)
 *   6. l = sum_t exp(s_t - m)  (+ exp(sink_h - m))
 *   7. out_d = sum_t exp(s_t - m) v_td / l ;  lse = m + log(l)
 *      (V3 "lse" restriction bullet: subtract the max, exponentiate, sum,
 *       add the log of the sum back to the max)
 *   8. no surviving t: out = 0, lse = +inf (V4 empty-tensor rule).
 *
 * Everything is double precision; fp16/bf16 inputs are widened exactly.
 * The output is left in double (unrounded); callers round as they need.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F16 = 0, OR_BF16 = 1, OR_I8 = 2 };

/* IEEE binary16 -> double, bit by bit. */
static double half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (exp == 0) {
        v = ldexp((double)man, -24);                  /* subnormal or zero */
    } else if (exp == 31) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp((double)(man | 0x400), exp - 25);
    }
    return sign ? -v : v;
}

/* bfloat16 is the top half of an IEEE binary32. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void *base, int dtype, int64_t idx) {
    switch (dtype) {
    case OR_F16: return half_to_double(((const uint16_t *)base)[idx]);
    case OR_BF16: return bf16_to_double(((const uint16_t *)base)[idx]);
    default: return (double)((const int8_t *)base)[idx];
    }
}

typedef struct {
    const void *q; int q_dtype;                 /* [nTokens, H, D]             */
    const void *k; const void *v; int kv_dtype; /* [numBlocks, bs, KVH, D]     */
    int64_t num_blocks; int bs;
    const int32_t *block_tables; int max_blocks;/* [B, max_blocks]             */
    const int32_t *seq_len; const int32_t *kv_seq_len; int batch;
    int H, KVH, D;
    double qk_scale; int mask_type;
    const float *slopes;                        /* [H] or NULL                 */
    const void *pse; int pse_dtype; int pse_maxq; int pse_maxkv; /* or NULL    */
    const float *sink;                          /* [H] or NULL                 */
    const float *k_scale, *k_offset, *v_scale, *v_offset; /* [KVH, D] or NULL  */
    int kv_layout;                              /* 0 BnBsH, 1 BnNBsD           */
    int k_mode, v_mode;                         /* 0 per-channel, 1 per-token  */
    int64_t k_tok_stride, v_tok_stride;         /* per-token: row stride S     */
    int band; int64_t pre_tokens, next_tokens;  /* band mask (sparseMode 4)    */
} oracle_args;

/* int8 dequantisation of cache value x of (sequence b, position t, channel
 * d, KV head kvh): scale * (x + offset) with scale/offset chosen by mode. */
static double dequant(const float *scale, const float *offset, int mode, int64_t tok_stride,
                      int b, int64_t t, int kvh, int D, int d, double x) {
    int64_t idx = mode == 1 ? (int64_t)b * tok_stride + t : (int64_t)kvh * D + d;
    double off = offset ? (double)offset[idx] : 0.0;
    return (double)scale[idx] * (x + off);
}

/* Element offset of cache row (blk, off) of KV head kvh. */
static int64_t cache_row(const oracle_args *a, int64_t blk, int off, int kvh) {
    if (a->kv_layout == 1)
        return ((blk * a->KVH + kvh) * a->bs + off) * (int64_t)a->D;
    return ((blk * a->bs + off) * a->KVH + kvh) * (int64_t)a->D;
}

/* One (b, i, h) row.  probs (optional) receives the normalised weight of each
 * logical position t < kvSeqLen[b] (0 where masked).  Returns the number of
 * surviving keys; -1 on an out-of-range block id. */
static int64_t oracle_row(const oracle_args *a, int b, int i, int h, int64_t token,
                          double *out, double *lse, double *probs) {
    const int g = a->H / a->KVH;
    const int kvh = h / g;
    const int D = a->D;
    const int64_t kvlen = a->kv_seq_len[b];
    const int64_t qpos = kvlen - (int64_t)a->seq_len[b] + i;
    const int causal = (a->mask_type == 9 || a->mask_type == 3);

    double *qv = (double *)malloc(sizeof(double) * D);
    double *s = (double *)malloc(sizeof(double) * (kvlen > 0 ? kvlen : 1));
    unsigned char *keep = (unsigned char *)malloc(kvlen > 0 ? kvlen : 1);
    for (int d = 0; d < D; ++d)
        qv[d] = load_elem(a->q, a->q_dtype, (token * a->H + h) * (int64_t)D + d);

    int64_t n_keep = 0;
    double m = -INFINITY;
    for (int64_t t = 0; t < kvlen; ++t) {
        keep[t] = 0;
        if (causal && t > qpos) continue;
        if (a->band && (t < qpos - a->pre_tokens || t > qpos + a->next_tokens)) continue;
        int32_t blk = a->block_tables[(int64_t)b * a->max_blocks + t / a->bs];
        if (blk < 0 || blk >= a->num_blocks) { free(qv); free(s); free(keep); return -1; }
        int64_t row = cache_row(a, blk, t % a->bs, kvh);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) {
            double kd = load_elem(a->k, a->kv_dtype, row + d);
            if (a->kv_dtype == OR_I8)
                kd = dequant(a->k_scale, a->k_offset, a->k_mode, a->k_tok_stride, b, t, kvh, D, d, kd);
            dot += qv[d] * kd;
        }
        double st = a->qk_scale * dot;
        if (a->mask_type == 3) st += (double)a->slopes[h] * (double)(t - qpos);
        if (a->pse) {
            int64_t pidx = (((int64_t)b * a->H + h) * a->pse_maxq + i) * (int64_t)a->pse_maxkv + t;
            st += load_elem(a->pse, a->pse_dtype, pidx);
        }
        s[t] = st;
        keep[t] = 1;
        ++n_keep;
        if (st > m) m = st;
    }

    if (n_keep == 0) {
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        *lse = INFINITY;
        if (probs) for (int64_t t = 0; t < kvlen; ++t) probs[t] = 0.0;
        free(qv); free(s); free(keep);
        return 0;
    }
    if (a->sink && (double)a->sink[h] > m) m = (double)a->sink[h];

    double l = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t t = 0; t < kvlen; ++t) {
        if (!keep[t]) continue;
        double p = exp(s[t] - m);
        s[t] = p;
        l += p;
        int32_t blk = a->block_tables[(int64_t)b * a->max_blocks + t / a->bs];
        int64_t row = cache_row(a, blk, t % a->bs, kvh);
        for (int d = 0; d < D; ++d) {
            double vd = load_elem(a->v, a->kv_dtype, row + d);
            if (a->kv_dtype == OR_I8)
                vd = dequant(a->v_scale, a->v_offset, a->v_mode, a->v_tok_stride, b, t, kvh, D, d, vd);
            out[d] += p * vd;
        }
    }
    if (a->sink) l += exp((double)a->sink[h] - m);
    for (int d = 0; d < D; ++d) out[d] /= l;
    *lse = m + log(l);
    if (probs)
        for (int64_t t = 0; t < kvlen; ++t) probs[t] = keep[t] ? s[t] / l : 0.0;
    free(qv); free(s); free(keep);
    return n_keep;
}

/*
 * Full attention, or a subset of rows.
 *   rows == NULL: every (token, head) row; out [nTokens, H, D], lse [nTokens, H].
 *   rows != NULL: n_rows pairs (token, head); out [n_rows, D], lse [n_rows].
 * Returns 0 on success, -1 on an out-of-range block id, -2 on bad arguments.
 */
int fia_oracle_attention(
    const void *q, int q_dtype, const void *k, const void *v, int kv_dtype,
    int64_t num_blocks, int bs, const int32_t *block_tables, int max_blocks,
    const int32_t *seq_len, const int32_t *kv_seq_len, int batch,
    int H, int KVH, int D, double qk_scale, int mask_type, const float *slopes,
    const void *pse, int pse_dtype, int pse_maxq, int pse_maxkv, const float *sink,
    const float *k_scale, const float *k_offset, const float *v_scale, const float *v_offset,
    const int64_t *rows, int64_t n_rows, int n_threads, double *out, double *lse, int kv_layout,
    int k_mode, int v_mode, int64_t k_tok_stride, int64_t v_tok_stride,
    int band, int64_t pre_tokens, int64_t next_tokens) {
    if (H <= 0 || KVH <= 0 || H % KVH != 0 || D <= 0 || bs <= 0) return -2;
    if (kv_layout != 0 && kv_layout != 1) return -2;
    if (k_mode < 0 || k_mode > 1 || v_mode < 0 || v_mode > 1) return -2;
    if (kv_dtype == OR_I8 && (!k_scale || !v_scale)) return -2;
    if (mask_type == 3 && !slopes) return -2;
    oracle_args a = {.q = q, .q_dtype = q_dtype, .k = k, .v = v, .kv_dtype = kv_dtype,
                     .num_blocks = num_blocks, .bs = bs, .block_tables = block_tables,
                     .max_blocks = max_blocks, .seq_len = seq_len, .kv_seq_len = kv_seq_len,
                     .batch = batch, .H = H, .KVH = KVH, .D = D, .qk_scale = qk_scale,
                     .mask_type = mask_type, .slopes = slopes, .pse = pse, .pse_dtype = pse_dtype,
                     .pse_maxq = pse_maxq, .pse_maxkv = pse_maxkv, .sink = sink,
                     .k_scale = k_scale, .k_offset = k_offset, .v_scale = v_scale,
                     .v_offset = v_offset, .kv_layout = kv_layout, .k_mode = k_mode,
                     .v_mode = v_mode, .k_tok_stride = k_tok_stride, .v_tok_stride = v_tok_stride,
                     .band = band, .pre_tokens = pre_tokens, .next_tokens = next_tokens};
    /* token -> (b, i) */
    int64_t n_tokens = 0;
    for (int b = 0; b < batch; ++b) n_tokens += seq_len[b];
    int32_t *tok_b = (int32_t *)malloc(sizeof(int32_t) * (n_tokens > 0 ? n_tokens : 1));
    int32_t *tok_i = (int32_t *)malloc(sizeof(int32_t) * (n_tokens > 0 ? n_tokens : 1));
    int64_t pos = 0;
    for (int b = 0; b < batch; ++b)
        for (int i = 0; i < seq_len[b]; ++i) { tok_b[pos] = b; tok_i[pos] = i; ++pos; }

    int64_t total = rows ? n_rows : n_tokens * H;
    int err = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 4) reduction(min : err)
#endif
    for (int64_t r = 0; r < total; ++r) {
        int64_t token = rows ? rows[2 * r] : r / H;
        int h = rows ? (int)rows[2 * r + 1] : (int)(r % H);
        if (token < 0 || token >= n_tokens || h < 0 || h >= H) { err = -2; continue; }
        int64_t st = oracle_row(&a, tok_b[token], tok_i[token], h, token,
                                out + r * (int64_t)D, lse + r, NULL);
        if (st < 0) err = -1;
    }
    free(tok_b);
    free(tok_i);
    return err;
}

/* Softmax weights of one row over the logical positions t < kvSeqLen[b]
 * (masked positions get 0).  Used to check the weights' invariants. */
int fia_oracle_row_probs(
    const void *q, int q_dtype, const void *k, const void *v, int kv_dtype,
    int64_t num_blocks, int bs, const int32_t *block_tables, int max_blocks,
    const int32_t *seq_len, const int32_t *kv_seq_len, int batch,
    int H, int KVH, int D, double qk_scale, int mask_type, const float *slopes,
    const void *pse, int pse_dtype, int pse_maxq, int pse_maxkv, const float *sink,
    const float *k_scale, const float *k_offset, const float *v_scale, const float *v_offset,
    int b, int i, int h, double *probs, double *out, double *lse, int kv_layout,
    int k_mode, int v_mode, int64_t k_tok_stride, int64_t v_tok_stride,
    int band, int64_t pre_tokens, int64_t next_tokens) {
    if (H <= 0 || KVH <= 0 || H % KVH != 0 || b < 0 || b >= batch) return -2;
    if (kv_layout != 0 && kv_layout != 1) return -2;
    if (k_mode < 0 || k_mode > 1 || v_mode < 0 || v_mode > 1) return -2;
    oracle_args a = {.q = q, .q_dtype = q_dtype, .k = k, .v = v, .kv_dtype = kv_dtype,
                     .num_blocks = num_blocks, .bs = bs, .block_tables = block_tables,
                     .max_blocks = max_blocks, .seq_len = seq_len, .kv_seq_len = kv_seq_len,
                     .batch = batch, .H = H, .KVH = KVH, .D = D, .qk_scale = qk_scale,
                     .mask_type = mask_type, .slopes = slopes, .pse = pse, .pse_dtype = pse_dtype,
                     .pse_maxq = pse_maxq, .pse_maxkv = pse_maxkv, .sink = sink,
                     .k_scale = k_scale, .k_offset = k_offset, .v_scale = v_scale,
                     .v_offset = v_offset, .kv_layout = kv_layout, .k_mode = k_mode,
                     .v_mode = v_mode, .k_tok_stride = k_tok_stride, .v_tok_stride = v_tok_stride,
                     .band = band, .pre_tokens = pre_tokens, .next_tokens = next_tokens};
    int64_t token = 0;
    for (int bb = 0; bb < b; ++bb) token += seq_len[bb];
    token += i;
    int64_t st = oracle_row(&a, b, i, h, token, out, lse, probs);
    return st < 0 ? -1 : 0;
}

int fia_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
