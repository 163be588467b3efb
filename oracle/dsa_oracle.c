/*
 * dsa_oracle.c -- plain, slow, single-threaded CPU oracle for the DeepSeek
 * Sparse Attention hot path (lightning indexer, top-k selection, sparse
 * latent attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; neither includes the other.
 *
 * Sources (web pages the method is taken from):
 *   [V32-IDX]  "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward excerpt:
 *              rotate_activation, act_quant,
 *              k cache write, weight fold, fp8_index, additive mask, topk.
 *   [V32-MASK] "DeepSeek-V3.2-Exp - Causal mask", Transformer.forward excerpt:
 *              with more than one new token, a mask that is -inf above the
 *              diagonal (future positions), none otherwise.
 *   [V32-MLA]  same page, MLA prefill excerpt: an index mask that is -inf except
 *              at the selected positions, plus the causal mask; softmax; value mix.
 *   [DIAG]     "DeepSeek Sparse Attention, one decode step in one layer (V3.2
 *              sizes)" diagram: I(t,s) = sum_j w_j ReLU(q_j . k_s), k = 2048,
 *              core attention in MQA mode over the selected latents, each latent
 *              row is key and value.
 *   [V4-CSA]   "visualize_attention_masks.py (DeepSeek-V4)", CSA branch: the
 *              indexer scores compressed entries (m tokens each, m the compress
 *              rate); an entry is causally available to the query at position i
 *              once its m tokens are in, i.e. entry < (i + 1) // m; the top-k
 *              lists entry ids and pads with -1 (warm-up sentinel).
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *   - rotate_activation: orthonormal Walsh-Hadamard transform in natural
 *     (Sylvester) order, butterflies in fp32 with stride 1, 2, 4, ..., then one
 *     multiply by fp32(D^-1/2).
 *   - act_quant: one block per D-vector; scale = max(amax, 1e-4) / 448 and
 *     y = e4m3(x / scale), both divisions correctly rounded fp32, e4m3 rounding
 *     to nearest even with saturation to +-448.
 *   - fp8_index: per-head dot products of the decoded FP8 values accumulated
 *     exactly (fp64), ReLU, weighted head sum in fp64, times the key scale,
 *     rounded once to fp32.
 *   - topk: ties broken towards the lower position; rows with fewer causal
 *     positions than k are padded with -1; the selection is written in
 *     ascending position order.
 *   - sparse attention: the latent row is [c (dc) | k_pe (dr)], the query is
 *     already in latent space; logits, softmax and the value mix in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* FP8 e4m3fn: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no     */
/* infinities, S.1111.111 is NaN, largest finite 448 = 1.75 * 2^8, smallest   */
/* subnormal 2^-9.                                                           */
/* ------------------------------------------------------------------------- */

double oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 7;
    double v;
    if (e == 0xF && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);             /* subnormal: m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x))
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0)                           /* satfinite */
        return sign | 0x7E;
    /* spacing of the e4m3 grid in the binade of a */
    double spacing;
    if (a < ldexp(1.0, -6)) {
        spacing = ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);                        /* a = f * 2^ex, f in [0.5, 1) */
        spacing = ldexp(1.0, (ex - 1) - 3);
    }
    double q = a / spacing;                   /* exact: power-of-two divisor */
    double r = nearbyint(q);                  /* default mode: nearest, ties to even */
    double v = r * spacing;
    if (v > 448.0)
        v = 448.0;
    if (v == 0.0)
        return sign;
    if (v < ldexp(1.0, -6))                   /* subnormal result */
        return sign | (uint8_t)(v / ldexp(1.0, -9));
    int ex;
    double f = frexp(v, &ex);                 /* v = f * 2^ex */
    int e = ex - 1;                           /* v = (2f) * 2^e, 2f in [1, 2) */
    int m = (int)((2.0 * f - 1.0) * 8.0);
    return sign | (uint8_t)(((e + 7) << 3) | m);
}

void oracle_e4m3_encode_array(const float *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------------- */
/* rotate_activation [V32-IDX]: Walsh-Hadamard rotation of one D-vector.      */
/* ------------------------------------------------------------------------- */

float oracle_hadamard_scale(int D)
{
    return (float)(1.0 / sqrt((double)D));
}

void oracle_fwht_f32(float *x, int D)
{
    for (int h = 1; h < D; h <<= 1) {
        for (int i = 0; i < D; i++) {
            if (i & h)
                continue;
            float a = x[i];
            float b = x[i + h];
            x[i] = a + b;
            x[i + h] = a - b;
        }
    }
    float sc = oracle_hadamard_scale(D);
    for (int i = 0; i < D; i++)
        x[i] = x[i] * sc;
}

/* act_quant [V32-IDX]: blockwise FP8 quantisation of n values. */
void oracle_act_quant(const float *x, int n, int block, uint8_t *y, float *scale)
{
    for (int b0 = 0; b0 < n; b0 += block) {
        float amax = 0.0f;
        for (int i = b0; i < b0 + block; i++) {
            float a = fabsf(x[i]);
            if (a > amax)
                amax = a;
        }
        float clamped = amax > 1e-4f ? amax : 1e-4f;
        float s = clamped / 448.0f;
        scale[b0 / block] = s;
        for (int i = b0; i < b0 + block; i++)
            y[i] = oracle_e4m3_encode(x[i] / s);
    }
}

/*
 * Indexer quantisation of n_vec D-vectors [V32-IDX]: rotate_activation then
 * act_quant with block = D.  Input vector v is x[v*D ...]; its codes go to
 * out[v*D ...] and its scale to scale[v].
 */
void oracle_indexer_quant(const float *x, int64_t n_vec, int D, uint8_t *out, float *scale)
{
    float *tmp = (float *)malloc(sizeof(float) * (size_t)D);
    for (int64_t v = 0; v < n_vec; v++) {
        memcpy(tmp, x + v * D, sizeof(float) * (size_t)D);
        oracle_fwht_f32(tmp, D);
        oracle_act_quant(tmp, D, D, out + v * D, scale + v);
    }
    free(tmp);
}

/*
 * Rotary embedding of the first R elements of one vector, not interleaved
 * [V32-IDX: the first rope_head_dim elements get the rotary embedding, not
 * interleaved, and are put back in front of the rest].  Element j and element j + R/2
 * (j < R/2) are the real and imaginary parts of one complex number, which is
 * multiplied by the position's unit complex cs[2j] + i cs[2j+1] (cos, sin of
 * frequency j): (x1 + i x2)(c + i s) = (x1 c - x2 s) + i (x1 s + x2 c), each
 * product and sum rounded to fp32.  Elements R .. D-1 are not touched.
 */
void oracle_rope_half(float *x, int R, const float *cs)
{
    int half = R / 2;
    for (int j = 0; j < half; j++) {
        float c = cs[2 * j], sn = cs[2 * j + 1];
        float x1 = x[j], x2 = x[j + half];
        float re_a = x1 * c, re_b = x2 * sn;
        float im_a = x1 * sn, im_b = x2 * c;
        x[j] = re_a - re_b;
        x[j + half] = im_a + im_b;
    }
}

/*
 * The ue8m0 scale format [V32-IDX: act_quant(x, block_size, scale_fmt)]: the
 * scale is stored as a bare power of two, here the smallest power of two not
 * below the fp32 scale max(amax, 1e-4) / 448, so that |x / scale| stays within
 * the e4m3 range.
 */
float oracle_scale_ue8m0(float s)
{
    int e;
    double m = frexp((double)s, &e);          /* s = m * 2^e, 0.5 <= m < 1 */
    if (m == 0.5)
        return s;
    return (float)ldexp(1.0, e);
}

/* act_quant with the scale format: fmt 0 = fp32 scale, 1 = ue8m0 scale. */
void oracle_act_quant_fmt(const float *x, int n, int block, int fmt, uint8_t *y, float *scale)
{
    for (int b0 = 0; b0 < n; b0 += block) {
        float amax = 0.0f;
        for (int i = b0; i < b0 + block; i++) {
            float a = fabsf(x[i]);
            if (a > amax)
                amax = a;
        }
        float clamped = amax > 1e-4f ? amax : 1e-4f;
        float s = clamped / 448.0f;
        if (fmt == 1)
            s = oracle_scale_ue8m0(s);
        scale[b0 / block] = s;
        for (int i = b0; i < b0 + block; i++)
            y[i] = oracle_e4m3_encode(x[i] / s);
    }
}

/*
 * The indexer's query and key preparation [V32-IDX, Indexer.forward]: for
 * every query head vector q[b, s, h, :] and key vector k[b, s, :] (D each, fp32):
 * rotary embedding of the first R elements with the angles of row s of cs
 * ([S][R/2][2], the caller's freqs_cis rows start_pos .. start_pos + S - 1),
 * rotate_activation, act_quant with block = D and the scale format fmt.
 * Query codes / scales go to q_fp8 [B,S,H,D] / q_scale [B,S,H]; key codes /
 * scales to k_fp8 [B,S,D] / k_scale [B,S] (the rows a cache append writes at
 * positions start_pos .. start_pos + S - 1).
 */
void oracle_indexer_prologue(const float *q, const float *k, int B, int S, int H, int D, int R,
                             const float *cs, int fmt, uint8_t *q_fp8, float *q_scale,
                             uint8_t *k_fp8, float *k_scale)
{
    float *tmp = (float *)malloc(sizeof(float) * (size_t)D);
    for (int b = 0; b < B; b++) {
        for (int s = 0; s < S; s++) {
            const float *cs_s = cs + (size_t)s * (size_t)R;
            for (int h = 0; h <= H; h++) {
                /* h < H: query head h; h == H: the key */
                int64_t v = ((int64_t)b * S + s) * H + h;
                const float *src = h < H ? q + v * D : k + ((int64_t)b * S + s) * D;
                memcpy(tmp, src, sizeof(float) * (size_t)D);
                oracle_rope_half(tmp, R, cs_s);
                oracle_fwht_f32(tmp, D);
                if (h < H)
                    oracle_act_quant_fmt(tmp, D, D, fmt, q_fp8 + v * D, q_scale + v);
                else
                    oracle_act_quant_fmt(tmp, D, D, fmt, k_fp8 + ((int64_t)b * S + s) * D,
                                         k_scale + (int64_t)b * S + s);
            }
        }
    }
    free(tmp);
}

/*
 * FP8 latent row [DIAG: "cache: latents (T x 576, FP8 + bf16 RoPE)", "Stored per
 * token per layer: 656 B latent row"].  The latent part c (the first dc values)
 * is quantised in blocks of 128 exactly as act_quant does (one fp32 scale per
 * block); the rotary part (the last dr values) stays bf16, rounded to nearest
 * even.  Row layout: [dc e4m3 codes | dc/128 fp32 scales | dr bf16 values],
 * 512 + 16 + 128 = 656 bytes at the V3.2 sizes.
 */
int64_t oracle_latent_row_bytes(int dc, int dr)
{
    return (int64_t)dc + (int64_t)(dc / 128) * 4 + (int64_t)dr * 2;
}

static uint16_t bf16_rne(float x)
{
    uint32_t b;
    memcpy(&b, &x, 4);
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu))
        return (uint16_t)((b >> 16) | 0x40);              /* quiet NaN */
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

void oracle_latent_quant(const float *x, int dc, int dr, uint8_t *row)
{
    int nb = dc / 128;
    float *sc = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    oracle_act_quant(x, dc, 128, row, sc);
    memcpy(row + dc, sc, sizeof(float) * (size_t)nb);
    for (int i = 0; i < dr; i++) {
        uint16_t h = bf16_rne(x[dc + i]);
        memcpy(row + dc + 4 * nb + 2 * i, &h, 2);
    }
    free(sc);
}

/* Decoded row: c[i] = e4m3(code_i) * scale[i / 128] (rounded to fp32), k_pe from bf16. */
void oracle_latent_dequant(const uint8_t *row, int dc, int dr, float *x)
{
    int nb = dc / 128;
    for (int i = 0; i < dc; i++) {
        float s;
        memcpy(&s, row + dc + 4 * (i / 128), 4);
        x[i] = (float)(oracle_e4m3_decode(row[i]) * (double)s);
    }
    for (int i = 0; i < dr; i++) {
        uint16_t h;
        memcpy(&h, row + dc + 4 * nb + 2 * i, 2);
        uint32_t b = (uint32_t)h << 16;
        memcpy(&x[dc + i], &b, 4);
    }
}

/*
 * Weight fold [V32-IDX]: weights * n_heads^-1/2, then * q_scale * softmax_scale,
 * each product in fp32 and in that order.
 */
float oracle_weight_fold(float w, int H, float q_scale, float softmax_scale)
{
    float hs = (float)(1.0 / sqrt((double)H));
    float t = w * hs;
    t = t * q_scale;
    t = t * softmax_scale;
    return t;
}

/*
 * fp8_index + additive causal mask [V32-IDX], [V32-MASK], [DIAG].
 *   q_fp8   [B,S,H,D]  codes of the rotated, quantised queries
 *   q_scale [B,S,H]
 *   w       [B,S,H]    raw per-head weights (weights_proj output)
 *   k_cache [B,t_max,D] codes, k_scale [B,t_max]
 *   scores  [B,S,T]    fp32; position t of query s is masked (-inf) when
 *                      t > start_pos + s.
 */
void oracle_index_scores(const uint8_t *q_fp8, const float *q_scale, const float *w,
                         const uint8_t *k_cache, const float *k_scale, int64_t t_max,
                         int B, int S, int H, int D, int64_t start_pos, int64_t T,
                         float softmax_scale, float *scores)
{
    double *wf = (double *)malloc(sizeof(double) * (size_t)H);
    double *qd = (double *)malloc(sizeof(double) * (size_t)H * (size_t)D);
    double *kd = (double *)malloc(sizeof(double) * (size_t)D);
    for (int b = 0; b < B; b++) {
        for (int s = 0; s < S; s++) {
            int64_t row = (int64_t)b * S + s;
            for (int h = 0; h < H; h++) {
                wf[h] = (double)oracle_weight_fold(w[row * H + h], H, q_scale[row * H + h],
                                                   softmax_scale);
                for (int d = 0; d < D; d++)
                    qd[h * D + d] = oracle_e4m3_decode(q_fp8[(row * H + h) * D + d]);
            }
            for (int64_t t = 0; t < T; t++) {
                float *dst = scores + row * T + t;
                if (t > start_pos + s) {
                    *dst = -INFINITY;
                    continue;
                }
                const uint8_t *kc = k_cache + ((int64_t)b * t_max + t) * D;
                for (int d = 0; d < D; d++)
                    kd[d] = oracle_e4m3_decode(kc[d]);
                double acc = 0.0;
                for (int h = 0; h < H; h++) {
                    double dot = 0.0;
                    for (int d = 0; d < D; d++)
                        dot += qd[h * D + d] * kd[d];
                    if (dot > 0.0)
                        acc += wf[h] * dot;
                }
                *dst = (float)(acc * (double)k_scale[(int64_t)b * t_max + t]);
            }
        }
    }
    free(wf);
    free(qd);
    free(kd);
}

/* ------------------------------------------------------------------------- */
/* topk [V32-IDX]: K = min(index_topk, end_pos) slots per query.              */
/* ------------------------------------------------------------------------- */

typedef struct {
    float score;
    int64_t pos;
} scored_pos;

static int by_score_desc_pos_asc(const void *pa, const void *pb)
{
    const scored_pos *a = (const scored_pos *)pa;
    const scored_pos *b = (const scored_pos *)pb;
    /* NaN sorts last */
    int an = isnan(a->score), bn = isnan(b->score);
    if (an != bn)
        return an - bn;
    if (!an) {
        if (a->score > b->score)
            return -1;
        if (a->score < b->score)
            return 1;
    }
    return (a->pos > b->pos) - (a->pos < b->pos);
}

static int by_pos_asc(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * One row: ranks positions 0 .. n_valid - 1 of `row` by (score desc, position
 * asc), keeps the first min(K, n_valid), writes them in ascending position
 * order into dst[0 .. K) and fills the remaining slots with -1.
 */
static void select_row(const float *row, int64_t n_valid, int K, scored_pos *buf, int32_t *dst)
{
    for (int64_t t = 0; t < n_valid; t++) {
        buf[t].score = row[t];
        buf[t].pos = t;
    }
    qsort(buf, (size_t)n_valid, sizeof(scored_pos), by_score_desc_pos_asc);
    int m = (int64_t)K < n_valid ? K : (int)n_valid;
    for (int j = 0; j < m; j++)
        dst[j] = (int32_t)buf[j].pos;
    qsort(dst, (size_t)m, sizeof(int32_t), by_pos_asc);
    for (int j = m; j < K; j++)
        dst[j] = -1;
}

/*
 * scores [B,S,T]; idx [B,S,K] with K = min(k, T).  Row (b,s) ranks the causal
 * positions t <= start_pos + s by (score desc, t asc), keeps the first
 * min(K, start_pos + s + 1), writes them in ascending position order and fills
 * the remaining slots with -1.
 */
void oracle_topk_select(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                        int k, int32_t *idx)
{
    int K = (int64_t)k < T ? k : (int)T;
    scored_pos *buf = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)(T > 0 ? T : 1));
    for (int64_t row = 0; row < (int64_t)B * S; row++) {
        int s = (int)(row % S);
        int64_t n_valid = start_pos + s + 1;
        if (n_valid > T)
            n_valid = T;
        select_row(scores + row * T, n_valid, K, buf, idx + row * K);
    }
    free(buf);
}

/* ------------------------------------------------------------------------- */
/* V4 compressed sparse attention (CSA) indexer [V4-CSA]                      */
/* ------------------------------------------------------------------------- */

/* Entries of m tokens available to the query at absolute position i. */
int64_t oracle_csa_available(int64_t i, int m)
{
    return (i + 1) / m;
}

/*
 * fp8_index over compressed entries: k_cache [B,t_max,D] / k_scale [B,t_max]
 * hold the entries' indexer keys (entry e at row e); scores [B,S,T] over
 * entries 0 .. T-1.  Every entry is scored as [V32-IDX]'s keys are (no mask),
 * then entry e of query s is masked (-inf) unless
 * e < oracle_csa_available(start_pos + s, m).
 */
void oracle_index_scores_csa(const uint8_t *q_fp8, const float *q_scale, const float *w,
                             const uint8_t *k_cache, const float *k_scale, int64_t t_max,
                             int B, int S, int H, int D, int64_t start_pos, int64_t T, int m,
                             float softmax_scale, float *scores)
{
    /* start_pos = T: every entry of every row is within the token-level causal
       limit, so nothing is masked there */
    oracle_index_scores(q_fp8, q_scale, w, k_cache, k_scale, t_max, B, S, H, D, T, T,
                        softmax_scale, scores);
    for (int64_t row = 0; row < (int64_t)B * S; row++) {
        int s = (int)(row % S);
        int64_t avail = oracle_csa_available(start_pos + s, m);
        for (int64_t e = avail < 0 ? 0 : avail; e < T; e++)
            scores[row * T + e] = -INFINITY;
    }
}

/*
 * Top-k over compressed entries: idx [B,S,K], K = min(k, T); row (b,s) keeps
 * the min(K, n_avail) best of its n_avail = min(T, available entries) by
 * (score desc, entry asc), in ascending entry order, padded with -1.
 */
void oracle_topk_select_csa(const float *scores, int B, int S, int64_t T, int64_t start_pos,
                            int m, int k, int32_t *idx)
{
    int K = (int64_t)k < T ? k : (int)T;
    scored_pos *buf = (scored_pos *)malloc(sizeof(scored_pos) * (size_t)(T > 0 ? T : 1));
    for (int64_t row = 0; row < (int64_t)B * S; row++) {
        int s = (int)(row % S);
        int64_t n_valid = oracle_csa_available(start_pos + s, m);
        if (n_valid > T)
            n_valid = T;
        if (n_valid < 0)
            n_valid = 0;
        select_row(scores + row * T, n_valid, K, buf, idx + row * K);
    }
    free(buf);
}

/* ------------------------------------------------------------------------- */
/* Sparse latent attention (MQA mode) [DIAG], semantics of [V32-MLA].         */
/* ------------------------------------------------------------------------- */

/*
 *   q   [B,S,Hq,dc+dr]   query in latent space, rotary part last
 *   kv  [B,t_max,dc+dr]  latent rows [c | k_pe]
 *   idx [B,S,k]          selected positions; -1 and positions after
 *                        start_pos + s (the causal mask) are skipped
 *   out [B,S,Hq,dc]      softmax(sm_scale * (q_c.c + q_r.k_pe)) mixed over c
 *   lse [B,S,Hq]         log-sum-exp of the logits (-inf when nothing is valid)
 */
void oracle_sparse_mla(const float *q, const float *kv, int64_t t_max, const int32_t *idx,
                       int B, int S, int Hq, int dc, int dr, int k, int64_t start_pos,
                       float sm_scale, float *out, float *lse)
{
    int dqk = dc + dr;
    double *z = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)dc);
    for (int b = 0; b < B; b++) {
        for (int s = 0; s < S; s++) {
            int64_t row = (int64_t)b * S + s;
            const int32_t *sel = idx + row * k;
            for (int h = 0; h < Hq; h++) {
                const float *qh = q + (row * Hq + h) * dqk;
                double m = -INFINITY;
                for (int j = 0; j < k; j++) {
                    int32_t i = sel[j];
                    if (i < 0 || (int64_t)i > start_pos + s) {
                        z[j] = -INFINITY;
                        continue;
                    }
                    const float *c = kv + ((int64_t)b * t_max + i) * dqk;
                    double dot = 0.0;
                    for (int d = 0; d < dc; d++)
                        dot += (double)qh[d] * (double)c[d];
                    for (int d = 0; d < dr; d++)
                        dot += (double)qh[dc + d] * (double)c[dc + d];
                    z[j] = (double)sm_scale * dot;
                    if (z[j] > m)
                        m = z[j];
                }
                float *oh = out + (row * Hq + h) * dc;
                if (m == -INFINITY) {
                    for (int d = 0; d < dc; d++)
                        oh[d] = 0.0f;
                    if (lse)
                        lse[row * Hq + h] = -INFINITY;
                    continue;
                }
                double l = 0.0;
                for (int d = 0; d < dc; d++)
                    o[d] = 0.0;
                for (int j = 0; j < k; j++) {
                    if (z[j] == -INFINITY)
                        continue;
                    double p = exp(z[j] - m);
                    l += p;
                    const float *c = kv + ((int64_t)b * t_max + sel[j]) * dqk;
                    for (int d = 0; d < dc; d++)
                        o[d] += p * (double)c[d];
                }
                for (int d = 0; d < dc; d++)
                    oh[d] = (float)(o[d] / l);
                if (lse)
                    lse[row * Hq + h] = (float)(m + log(l));
            }
        }
    }
    free(z);
    free(o);
}
