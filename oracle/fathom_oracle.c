/*
 * fathom_oracle.c -- plain, slow CPU oracle for the Fathom per-query
 * read-depth top-k key scan.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file.  It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never calls it.
 *
 * Source: "Fathom：面向卸载 KV 缓存稀疏解码的每查询读取深度" (the
 * papers.ananclaw.com explainer of arXiv 2609.17652), section 核心方法
 * (method): 存储侧 (storage side) and 读侧 (read side), and its simplified
 * reverse water-filling walk; plus the method summary on the proomt.com page
 * ("Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
 * Caches", Summary).  Every choice the pages leave open is a stated reading:
 *
 *   quantiser   per (head, channel) asymmetric min/max over all n keys,
 *               scale = (max-min)/L with L = 2^b - 1 levels for a b-bit K
 *               cache (b = 4; b = 8 for the 8-plane variant the page's
 *               部署前必读 item 3 asks for when the upstream K is 8-bit),
 *               code = clamp(floor((k-min)/scale+0.5), 0, L) in float32
 *               round-to-nearest with no fused ops; a constant channel
 *               gets scale 0 and code 0.
 *   planes      bit p of a code (p = 0 least significant, as on the page)
 *               is stored in slot b-1-p, so reading slots 0..t-1 reads the
 *               t most significant bits ("the first t planes are the t-bit
 *               quantiser" only holds MSB-first).
 *   variance    sigma^2 = population variance of the dequantised keys,
 *               from exact integer sums of codes.
 *   importance  w_c = (q_c*q_c)*sigma^2_c in float32, q widened from bf16.
 *   plan        channels in order of (w descending, channel ascending); each
 *               takes min(b, remaining budget) bits until the budget is
 *               spent, so channels of zero importance still take leftovers.
 *   score       reading t bits gives u = code >> (b-t); the key is rebuilt
 *               at the middle of that coarse bin and dotted with q in fp64.
 *   top-k       score descending, ties to the lower key index.
 *
 * Parity unpinned: recall against the exact top-k is a quality number only;
 * the pages print no recall to check it against.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared -lm.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define FO_OK 0
#define FO_ERR_ARG 1
#define FO_ERR_NONFINITE 3

/* Planes per channel: b = 4 for the 4-bit K cache; the oracle takes any
 * b in 1..8 so that the 8-plane variant is the same code. */
static int fo_bits_ok(int64_t bits) { return bits >= 1 && bits <= 8; }

/* ------------------------------------------------------------------ */
/* Storage side: b-bit quantisation of each channel.                    */
/* ------------------------------------------------------------------ */

/* keys: float32 [H][n][d] (token-major, as a K cache holds them).
 * Outputs: mn, scale float32 [H][d]; codes uint8 [H][d][n] (channel-major). */
int fo_quantize(const float *keys, int64_t H, int64_t n, int64_t d, int64_t bits,
                float *mn, float *scale, uint8_t *codes)
{
    if (H <= 0 || n <= 0 || d <= 0 || !fo_bits_ok(bits)) return FO_ERR_ARG;
    const int levels = (1 << bits) - 1;
    for (int64_t h = 0; h < H; ++h) {
        const float *kh = keys + h * n * d;
        for (int64_t c = 0; c < d; ++c) {
            float lo = kh[c], hi = kh[c];
            for (int64_t j = 0; j < n; ++j) {
                float x = kh[j * d + c];
                if (!isfinite(x)) return FO_ERR_NONFINITE;
                if (x < lo) lo = x;
                if (x > hi) hi = x;
            }
            uint8_t *out = codes + (h * d + c) * n;
            mn[h * d + c] = lo;
            if (hi == lo) {
                scale[h * d + c] = 0.0f;
                memset(out, 0, (size_t)n);
                continue;
            }
            float sc = (hi - lo) / (float)levels;
            scale[h * d + c] = sc;
            for (int64_t j = 0; j < n; ++j) {
                float diff = kh[j * d + c] - lo;
                float ratio = diff / sc;
                float shifted = ratio + 0.5f;
                float level = floorf(shifted);
                int v = (int)level;
                if (v < 0) v = 0;
                if (v > levels) v = levels;
                out[j] = (uint8_t)v;
            }
        }
    }
    return FO_OK;
}

/* Channel-major bit planes: planes uint32 [H][d][b][n_words]; slot s holds
 * bit (b-1-s) of the code; bit i of word w belongs to key 32*w+i; words
 * past the last key are zero.  n_words >= ceil(n/32). */
int fo_pack_planes(const uint8_t *codes, int64_t H, int64_t n, int64_t d, int64_t bits,
                   int64_t n_words, uint32_t *planes)
{
    if (n_words * 32 < n || !fo_bits_ok(bits)) return FO_ERR_ARG;
    memset(planes, 0, (size_t)(H * d * bits * n_words) * sizeof(uint32_t));
    for (int64_t h = 0; h < H; ++h)
        for (int64_t c = 0; c < d; ++c) {
            const uint8_t *cc = codes + (h * d + c) * n;
            uint32_t *pc = planes + (h * d + c) * bits * n_words;
            for (int64_t j = 0; j < n; ++j)
                for (int p = 0; p < bits; ++p)
                    if ((cc[j] >> p) & 1u)
                        pc[(bits - 1 - p) * n_words + j / 32] |= 1u << (j % 32);
        }
    return FO_OK;
}

/* Append m keys per KV head to an index holding n keys: the decode step's
 * new keys enter the b-bit K cache the explainer's read side scans
 * (核心方法 / 存储侧; the cache comes from the serving stack, 适用边界).
 * Reading: the new keys are quantised with the index's existing mn and
 * scale, in the quantiser's own float32 steps, and the level is clamped to
 * 0..2^b-1 (a key outside the stored range takes the nearest level); their
 * bits go to key positions n..n+m-1 of the planes; S1 and S2 grow by the
 * new codes and sigma^2 is recomputed from them with n+m keys.
 * clamped[h][c] (may be NULL) is incremented once per new key whose level
 * fell outside 0..2^b-1 (for a constant channel: any key other than mn), the
 * measure of range drift a caller re-quantises on.
 * keys float32 [H][m][d]; planes [H][d][b][n_words], 32*n_words >= n+m,
 * words past key n zero. */
int fo_append(const float *keys, int64_t H, int64_t n, int64_t m, int64_t d, int64_t bits,
              int64_t n_words, const float *mn, const float *scale, uint32_t *planes,
              int64_t *s1, int64_t *s2, float *sigma2, uint32_t *clamped)
{
    if (H <= 0 || n < 0 || m <= 0 || d <= 0 || n_words * 32 < n + m || !fo_bits_ok(bits))
        return FO_ERR_ARG;
    const int levels = (1 << bits) - 1;
    for (int64_t h = 0; h < H; ++h)
        for (int64_t c = 0; c < d; ++c) {
            const int64_t hc = h * d + c;
            const float lo = mn[hc], sc = scale[hc];
            uint32_t *pc = planes + hc * bits * n_words;
            for (int64_t i = 0; i < m; ++i) {
                const float x = keys[(h * m + i) * d + c];
                if (!isfinite(x)) return FO_ERR_NONFINITE;
                int v;
                int out_of_range;
                if (sc == 0.0f) {
                    v = 0;
                    out_of_range = x != lo;
                } else {
                    float diff = x - lo;
                    float ratio = diff / sc;
                    float shifted = ratio + 0.5f;
                    float level = floorf(shifted);
                    out_of_range = level < 0.0f || level > (float)levels;
                    v = level < 0.0f ? 0 : (level > (float)levels ? levels : (int)level);
                }
                const int64_t j = n + i;
                for (int p = 0; p < bits; ++p)
                    if ((v >> p) & 1)
                        pc[(bits - 1 - p) * n_words + j / 32] |= 1u << (j % 32);
                s1[hc] += v;
                s2[hc] += (int64_t)v * v;
                if (clamped && out_of_range) clamped[hc] += 1;
            }
            const int64_t nn = n + m;
            const int64_t num = nn * s2[hc] - s1[hc] * s1[hc];
            const double sd = (double)sc;
            sigma2[hc] = (float)((sd * sd) * ((double)num / ((double)nn * (double)nn)));
        }
    return FO_OK;
}

/* Inverse of fo_pack_planes (reads all b slots). */
int fo_unpack_planes(const uint32_t *planes, int64_t H, int64_t n, int64_t d, int64_t bits,
                     int64_t n_words, uint8_t *codes)
{
    if (n_words * 32 < n || !fo_bits_ok(bits)) return FO_ERR_ARG;
    for (int64_t h = 0; h < H; ++h)
        for (int64_t c = 0; c < d; ++c) {
            const uint32_t *pc = planes + (h * d + c) * bits * n_words;
            uint8_t *cc = codes + (h * d + c) * n;
            for (int64_t j = 0; j < n; ++j) {
                int v = 0;
                for (int p = 0; p < bits; ++p)
                    v |= (int)((pc[(bits - 1 - p) * n_words + j / 32] >> (j % 32)) & 1u) << p;
                cc[j] = (uint8_t)v;
            }
        }
    return FO_OK;
}

/* Per-channel statistics of the stored b-bit keys: S1 = sum code,
 * S2 = sum code^2 (exact int64) and the population variance of the
 * dequantised keys mn + scale*code:
 *   sigma^2 = scale^2 * (n*S2 - S1^2) / n^2,
 * evaluated as (double)(scale*scale) * ((double)num / ((double)n*n)),
 * then rounded to float32. */
int fo_channel_stats(const uint8_t *codes, int64_t H, int64_t n, int64_t d,
                     const float *scale, int64_t *s1, int64_t *s2, float *sigma2)
{
    for (int64_t h = 0; h < H; ++h)
        for (int64_t c = 0; c < d; ++c) {
            const uint8_t *cc = codes + (h * d + c) * n;
            int64_t a = 0, b = 0;
            for (int64_t j = 0; j < n; ++j) {
                a += cc[j];
                b += (int64_t)cc[j] * cc[j];
            }
            s1[h * d + c] = a;
            s2[h * d + c] = b;
            int64_t num = n * b - a * a;
            double sc = (double)scale[h * d + c];
            double sc2 = sc * sc;
            double nn = (double)n * (double)n;
            double frac = (double)num / nn;
            sigma2[h * d + c] = (float)(sc2 * frac);
        }
    return FO_OK;
}

/* Grouped per-token-block scales: the keys of a channel are cut into
 * blocks of `block` tokens, each quantised on its own (its own mn, scale,
 * S1, S2; the last block may hold fewer keys), the grouping quantised K
 * caches of serving stacks use (the explainer, 亮点 and 适用边界: the index
 * is the serving stack's quantised K).  sigma^2 stays one number per
 * channel: the population variance of all n dequantised keys, combined
 * from the blocks' exact sums in fp64, block by block in order, with the
 * pairwise update of Chan, Golub and LeVeque (1979):
 *   mean_b = mn_b + scale_b * (S1_b / n_b)
 *   M2_b   = (scale_b * scale_b) * ((n_b*S2_b - S1_b^2) / n_b)
 *   N' = N + n_b;  delta = mean_b - mean;  mean += delta * (n_b / N');
 *   M2 += M2_b + (delta * delta) * ((N * n_b) / N');  N = N'
 *   sigma^2 = (float)(M2 / n).
 * mn, scale float [nb][d]; s1, s2 int64 [nb][d] of one KV head;
 * sigma2 float [d]. */
int fo_blocked_sigma2(const float *mn, const float *scale, const int64_t *s1, const int64_t *s2,
                      int64_t d, int64_t n, int64_t block, float *sigma2)
{
    if (d <= 0 || n <= 0 || block <= 0) return FO_ERR_ARG;
    const int64_t nb = (n + block - 1) / block;
    for (int64_t c = 0; c < d; ++c) {
        double N = 0.0, mean = 0.0, M2 = 0.0;
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t nbk = (b + 1) * block <= n ? block : n - b * block;
            const int64_t i = b * d + c;
            const double nbd = (double)nbk;
            const double sc = (double)scale[i];
            const double mean_b = (double)mn[i] + sc * ((double)s1[i] / nbd);
            const int64_t num = nbk * s2[i] - s1[i] * s1[i];
            const double m2_b = (sc * sc) * ((double)num / nbd);
            const double Nn = N + nbd;
            const double delta = mean_b - mean;
            mean = mean + delta * (nbd / Nn);
            M2 = M2 + m2_b + (delta * delta) * ((N * nbd) / Nn);
            N = Nn;
        }
        sigma2[c] = (float)(M2 / (double)n);
    }
    return FO_OK;
}

/* ------------------------------------------------------------------ */
/* Read side: importance, reverse water-filling, union, bytes.          */
/* ------------------------------------------------------------------ */

static float bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* w_c = (q_c * q_c) * sigma^2_c, float32. */
int fo_importance(const uint16_t *q_bf16, const float *sigma2, int64_t d, float *w)
{
    for (int64_t c = 0; c < d; ++c) {
        float qc = bf16_value(q_bf16[c]);
        float qq = qc * qc;
        float wc = qq * sigma2[c];
        if (!isfinite(wc)) return FO_ERR_NONFINITE;
        w[c] = wc;
    }
    return FO_OK;
}

typedef struct { float key; int64_t c; } fo_rank_item;

/* (key descending, channel ascending) */
static int fo_rank_cmp(const void *pa, const void *pb)
{
    const fo_rank_item *a = (const fo_rank_item *)pa, *b = (const fo_rank_item *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->c < b->c) ? -1 : (a->c > b->c);
}

/* Reverse water-filling: visit channels from the most important down and
 * give each min(b, remaining) bits; once the budget is gone the rest get 0.
 * B must lie in [0, b*d]. */
int fo_plan_greedy(const float *w, int64_t d, int64_t B, int64_t bits, uint8_t *t)
{
    if (!fo_bits_ok(bits) || B < 0 || B > bits * d) return FO_ERR_ARG;
    fo_rank_item *order = (fo_rank_item *)malloc((size_t)d * sizeof *order);
    if (!order) return FO_ERR_ARG;
    for (int64_t c = 0; c < d; ++c) {
        if (!isfinite(w[c])) { free(order); return FO_ERR_NONFINITE; }
        order[c].key = w[c];
        order[c].c = c;
    }
    qsort(order, (size_t)d, sizeof *order, fo_rank_cmp);
    int64_t left = B;
    for (int64_t i = 0; i < d; ++i) {
        int64_t take = 0;
        if (left > 0) {
            take = left < bits ? left : bits;
            left -= take;
        }
        t[order[i].c] = (uint8_t)take;
    }
    free(order);
    return FO_OK;
}

/* Marginal-gain plan (a finer reverse water-filling for continuous
 * importance; the explainer's simplified walk hands out whole 4-bit
 * channels, 核心方法 / 读侧, and notes that finer handling is possible).
 * Reading: the distortion of a channel read at t bits falls as 4^-t, so
 * bit t+1 of channel c is worth w_c * 4^-t; the B bits go one at a time to
 * the channel of largest w_c * 4^-t_c (t_c < b), ties to the lower channel.
 * 4^-t is a power of two, so the float gains are exact.  B in [0, b*d]. */
int fo_plan_marginal(const float *w, int64_t d, int64_t B, int64_t bits, uint8_t *t)
{
    if (!fo_bits_ok(bits) || B < 0 || B > bits * d) return FO_ERR_ARG;
    for (int64_t c = 0; c < d; ++c) {
        if (!isfinite(w[c])) return FO_ERR_NONFINITE;
        t[c] = 0;
    }
    for (int64_t b = 0; b < B; ++b) {
        int64_t best = -1;
        float best_gain = 0.0f;
        for (int64_t c = 0; c < d; ++c) {
            if (t[c] >= bits) continue;
            const float gain = w[c] * (1.0f / (float)(1 << (2 * t[c])));
            if (best < 0 || gain > best_gain) {
                best = c;
                best_gain = gain;
            }
        }
        t[best] += 1;
    }
    return FO_OK;
}

/* Fixed-width baseline plan: the r channels of largest |q_c| (ties to the
 * lower channel) are read at all b bits, the rest not at all. */
int fo_fixed_plan(const uint16_t *q_bf16, int64_t d, int64_t r, int64_t bits, uint8_t *t)
{
    if (r < 0 || r > d || !fo_bits_ok(bits)) return FO_ERR_ARG;
    fo_rank_item *order = (fo_rank_item *)malloc((size_t)d * sizeof *order);
    if (!order) return FO_ERR_ARG;
    for (int64_t c = 0; c < d; ++c) {
        order[c].key = fabsf(bf16_value(q_bf16[c]));
        order[c].c = c;
    }
    qsort(order, (size_t)d, sizeof *order, fo_rank_cmp);
    for (int64_t i = 0; i < d; ++i) t[order[i].c] = (uint8_t)(i < r ? bits : 0);
    free(order);
    return FO_OK;
}

/* GQA union: planes are nested MSB-first, so a KV head that serves G query
 * heads reads T_c = max_g t_c^(g) planes of channel c. */
void fo_union(const uint8_t *t, int64_t G, int64_t d, uint8_t *T)
{
    for (int64_t c = 0; c < d; ++c) {
        uint8_t m = 0;
        for (int64_t g = 0; g < G; ++g)
            if (t[g * d + c] > m) m = t[g * d + c];
        T[c] = m;
    }
}

/* Bytes read = sum_c t_c * bytes_per_plane, one plane being n_words*4 bytes. */
uint64_t fo_plan_bytes(const uint8_t *t, int64_t d, int64_t n_words)
{
    uint64_t total = 0;
    for (int64_t c = 0; c < d; ++c) total += (uint64_t)t[c] * (uint64_t)n_words * 4u;
    return total;
}

/* ------------------------------------------------------------------ */
/* Scoring from the selected planes.                                    */
/* ------------------------------------------------------------------ */

/* A key read at t of b bits with value u = code >> (b-t) lies in the coarse
 * bin of fine levels [u*2^(b-t), u*2^(b-t) + 2^(b-t) - 1]; it is rebuilt at
 * the bin's middle.  t = b gives mn + scale*code; t = 0 gives
 * mn + scale*(2^b-1)/2 (7.5*scale for b = 4). */
static double fo_coarse_midpoint(float mn, float scale, int t, int u, int bits)
{
    int width = 1 << (bits - t);
    double level = (double)(width * u) + (double)(width - 1) / 2.0;
    return (double)mn + (double)scale * level;
}

/* Score every key of one KV head for one query from its plan t:
 * planes_h uint32 [d][b][n_words]; mn, scale [d]; q bf16 [d]; t [d];
 * s float64 [n].  Reads slots 0..t_c-1 of each channel (MSB first). */
int fo_score_planes(const uint32_t *planes_h, const float *mn, const float *scale,
                    const uint16_t *q_bf16, const uint8_t *t, int64_t d, int64_t bits,
                    int64_t n, int64_t n_words, double *s)
{
    if (!fo_bits_ok(bits)) return FO_ERR_ARG;
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) {
            int tc = t[c];
            if (tc < 0 || tc > bits) return FO_ERR_ARG;
            int u = 0;
            for (int slot = 0; slot < tc; ++slot) {
                uint32_t word = planes_h[(c * bits + slot) * n_words + j / 32];
                u = (u << 1) | (int)((word >> (j % 32)) & 1u);
            }
            acc += (double)bf16_value(q_bf16[c]) *
                   fo_coarse_midpoint(mn[c], scale[c], tc, u, (int)bits);
        }
        s[j] = acc;
    }
    return FO_OK;
}

/* The same score from the b-bit codes by re-quantising to t bits:
 * codes_h uint8 [d][n]. */
int fo_score_codes(const uint8_t *codes_h, const float *mn, const float *scale,
                   const uint16_t *q_bf16, const uint8_t *t, int64_t d, int64_t bits,
                   int64_t n, double *s)
{
    if (!fo_bits_ok(bits)) return FO_ERR_ARG;
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) {
            int tc = t[c];
            if (tc < 0 || tc > bits) return FO_ERR_ARG;
            int u = codes_h[c * n + j] >> (bits - tc);
            acc += (double)bf16_value(q_bf16[c]) *
                   fo_coarse_midpoint(mn[c], scale[c], tc, u, (int)bits);
        }
        s[j] = acc;
    }
    return FO_OK;
}

/* sum_c |q_c * khat_c,j| for the same reading: the scale a score's
 * rounding error is measured against. */
int fo_score_abs_planes(const uint32_t *planes_h, const float *mn, const float *scale,
                        const uint16_t *q_bf16, const uint8_t *t, int64_t d, int64_t bits,
                        int64_t n, int64_t n_words, double *a)
{
    if (!fo_bits_ok(bits)) return FO_ERR_ARG;
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) {
            int tc = t[c];
            if (tc < 0 || tc > bits) return FO_ERR_ARG;
            int u = 0;
            for (int slot = 0; slot < tc; ++slot) {
                uint32_t word = planes_h[(c * bits + slot) * n_words + j / 32];
                u = (u << 1) | (int)((word >> (j % 32)) & 1u);
            }
            acc += fabs((double)bf16_value(q_bf16[c]) *
                        fo_coarse_midpoint(mn[c], scale[c], tc, u, (int)bits));
        }
        a[j] = acc;
    }
    return FO_OK;
}

/* Exact score against the full-precision keys: keys_h float32 [n][d]. */
void fo_exact_scores(const float *keys_h, const uint16_t *q_bf16, int64_t n, int64_t d,
                     double *s)
{
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c)
            acc += (double)bf16_value(q_bf16[c]) * (double)keys_h[j * d + c];
        s[j] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* Top-k: a full sort.                                                  */
/* ------------------------------------------------------------------ */

typedef struct { double s; int64_t j; } fo_score_item;

static int fo_score_cmp(const void *pa, const void *pb)
{
    const fo_score_item *a = (const fo_score_item *)pa, *b = (const fo_score_item *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

/* The k keys of largest score, in order (score descending, index ascending). */
int fo_topk(const double *s, int64_t n, int64_t k, int32_t *idx, double *top_s)
{
    if (k < 1 || k > n) return FO_ERR_ARG;
    fo_score_item *items = (fo_score_item *)malloc((size_t)n * sizeof *items);
    if (!items) return FO_ERR_ARG;
    for (int64_t j = 0; j < n; ++j) {
        if (!isfinite(s[j])) { free(items); return FO_ERR_NONFINITE; }
        items[j].s = s[j];
        items[j].j = j;
    }
    qsort(items, (size_t)n, sizeof *items, fo_score_cmp);
    for (int64_t i = 0; i < k; ++i) {
        idx[i] = (int32_t)items[i].j;
        if (top_s) top_s[i] = items[i].s;
    }
    free(items);
    return FO_OK;
}

/* ------------------------------------------------------------------ */
/* After the scan: attention over the selected keys.                    */
/* ------------------------------------------------------------------ */

/* Softmax attention of one query over the keys listed in idx (the top-k the
 * scan selected; the explainer scores keys to decide which K/V to fetch for
 * sparse decoding, 解决什么真问题): logits l_i = scale * (q . K[idx_i]) with
 * q the bf16 query widened exactly, p = softmax(l) (max subtracted), out =
 * sum_i p_i V[idx_i]; all in fp64.  idx = NULL attends to all n keys (the
 * dense reference of the attention-error metric).
 * keys_h, values_h float32 [n][d]; out [d]. */
int fo_attention(const float *keys_h, const float *values_h, int64_t n, int64_t d,
                 const uint16_t *q_bf16, const int32_t *idx, int64_t k, double scale,
                 double *out)
{
    const int64_t cnt = idx ? k : n;
    if (cnt < 1 || d < 1) return FO_ERR_ARG;
    double *logit = (double *)malloc((size_t)cnt * sizeof *logit);
    if (!logit) return FO_ERR_ARG;
    double mx = -INFINITY;
    for (int64_t i = 0; i < cnt; ++i) {
        const int64_t j = idx ? idx[i] : i;
        if (j < 0 || j >= n) { free(logit); return FO_ERR_ARG; }
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c)
            acc += (double)bf16_value(q_bf16[c]) * (double)keys_h[j * d + c];
        logit[i] = scale * acc;
        if (logit[i] > mx) mx = logit[i];
    }
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    double denom = 0.0;
    for (int64_t i = 0; i < cnt; ++i) {
        const int64_t j = idx ? idx[i] : i;
        const double p = exp(logit[i] - mx);
        denom += p;
        for (int64_t c = 0; c < d; ++c) out[c] += p * (double)values_h[j * d + c];
    }
    for (int64_t c = 0; c < d; ++c) out[c] /= denom;
    free(logit);
    return FO_OK;
}

/* ------------------------------------------------------------------ */
/* One KV head's keys split across devices: merging the shards' top-k.  */
/* ------------------------------------------------------------------ */

/* Exact top-k of the union of S shard lists of one query: shard s holds
 * keys [offset_s, offset_s + n_s) and lists k_s of them (local index,
 * score).  Keys rank by (score descending, global index ascending), the
 * order the single-device top-k uses, so when each shard list is that
 * shard's top-k the merge is the top-k of all keys.  out_idx receives the k
 * global indices in ascending order, out_score their scores.
 * idx, score: [S][k_s]; offset: [S]. */
int fo_merge_topk(const int32_t *idx, const double *score, const int64_t *offset, int64_t S,
                  int64_t k_s, int64_t k, int32_t *out_idx, double *out_score)
{
    const int64_t m = S * k_s;
    if (S < 1 || k_s < 1 || k < 1 || k > m) return FO_ERR_ARG;
    fo_score_item *items = (fo_score_item *)malloc((size_t)m * sizeof *items);
    if (!items) return FO_ERR_ARG;
    for (int64_t s = 0; s < S; ++s)
        for (int64_t i = 0; i < k_s; ++i) {
            items[s * k_s + i].s = score[s * k_s + i];
            items[s * k_s + i].j = offset[s] + idx[s * k_s + i];
        }
    qsort(items, (size_t)m, sizeof *items, fo_score_cmp);
    /* the k best, then ascending global index (insertion sort: k is small) */
    for (int64_t i = 1; i < k; ++i) {
        fo_score_item x = items[i];
        int64_t p = i - 1;
        while (p >= 0 && items[p].j > x.j) { items[p + 1] = items[p]; --p; }
        items[p + 1] = x;
    }
    for (int64_t i = 0; i < k; ++i) {
        out_idx[i] = (int32_t)items[i].j;
        out_score[i] = items[i].s;
    }
    free(items);
    return FO_OK;
}
