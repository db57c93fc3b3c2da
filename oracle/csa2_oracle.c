/*
 * csa2_oracle.c -- plain CPU oracle of the CSA2 global-attention decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA path is compared
 * against.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load it; the product library never links, calls or
 * includes anything from here, and this file includes nothing of the product.
 *
 * Source of every rule below: the DeepSeek V4.1 Flash pages ("DeepSeek V4.1
 * Flash: architecture study notes", macin.top; "DeepSeek V4.1 Flash goes
 * online", myzaker).  Where those pages are silent, the reading taken is the
 * one stated next to the function and listed in the design notes.
 *
 * Precision: the two quantisers and the index score are defined in fp32 (the
 * kernel's precision: they decide integers -- codes, and Top-K membership),
 * evaluated here in a fixed order with explicit fmaf and no contraction
 * (build with -ffp-contract=off).  Dequantisation and attention are fp64.
 *
 * Parity status: every function here is pinned by tests (value tables, exact
 * rational evaluation of the fp32 order, brute-force sorts, dense-softmax
 * special cases).  Nothing is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
EXPORT float csa2o_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest with ties to even (NaN stays a quiet NaN).  On the
 * bit pattern: add half of the dropped range minus one, plus the kept lsb, then
 * drop the low 16 bits. */
EXPORT uint16_t csa2o_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* E2M1 (study notes, section 4 "main KV from FP8 to FP4": 4-bit E2M1 values).
 * Code = sign(1) | exponent(2) | mantissa(1); magnitudes by code 0..7. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

EXPORT double csa2o_e2m1_value(int code) {
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* E4M3 (the 8-bit per-16-channel scale of the same section; also the FP8
 * format of the SWA window and the indexer K).  Exponent bias 7, subnormals,
 * no infinities; 0x7F / 0xFF are NaN; largest finite 448. */
EXPORT double csa2o_e4m3_value(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round-to-nearest, ties to the even code, saturating to +-6 (reading: RNE
 * with saturation; no stochastic rounding at inference).  The sign of the
 * input is kept, so -0 and negative values that round to zero give code 0x8. */
EXPORT int csa2o_e2m1_encode(float r) {
    int sign = signbit(r) ? 8 : 0;
    double a = fabs((double)r);
    if (a >= 6.0) return sign | 7;
    int best = 0;
    double bd = a;
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - E2M1_MAG[c]);
        if (d < bd || (d == bd && (c & 1) == 0)) { best = c; bd = d; }
    }
    return sign | best;
}

/* E4M3 values of codes 0..255, filled once from csa2o_e4m3_value (speed only). */
static double E4M3_TAB[256];
static int e4m3_tab_ready = 0;

static void e4m3_tab_init(void) {
    if (e4m3_tab_ready) return;
#pragma omp critical(csa2o_e4m3_tab)
    {
        if (!e4m3_tab_ready) {
            for (int c = 0; c < 256; ++c) E4M3_TAB[c] = csa2o_e4m3_value(c);
            e4m3_tab_ready = 1;
        }
    }
}

/* Round-to-nearest-even into E4M3 with saturation to +-448; sign kept. */
EXPORT int csa2o_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    e4m3_tab_init();
    int sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double bd = a;
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - E4M3_TAB[c]);
        if (d < bd || (d == bd && (c & 1) == 0)) { best = c; bd = d; }
    }
    return sign | best;
}

/* ------------------------------------------------------------------------ */
/* a1: FP4 quantisation of main-KV entries                                   */
/* ------------------------------------------------------------------------ */
/* Study notes section 4 and myzaker "cache precision": every value is a 4-bit
 * E2M1 code, every 16 channels share one 8-bit E4M3 scale (4 + 8/16 = 4.5
 * bits per value), and there is no second, global scale.
 * Readings: scale = E4M3_RNE(amax / 6) in fp32; code_c = E2M1_RNE(x_c / scale)
 * with fp32 division; a group whose scale is zero stores all codes 0x0; two
 * codes per byte, the even channel in the low nibble.
 * x: bf16 bits [rows][width]; codes [rows][width/2]; scales [rows][width/16]. */
EXPORT void csa2o_quantize_fp4(const uint16_t *x, int64_t rows, int width,
                               uint8_t *codes, uint8_t *scales) {
    e4m3_tab_init();
#pragma omp parallel for schedule(static) if (rows > 256)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * width;
        for (int g = 0; g < width / 16; ++g) {
            float v[16];
            float amax = 0.0f;
            for (int c = 0; c < 16; ++c) {
                v[c] = csa2o_bf16_to_f32(xr[16 * g + c]);
                float a = fabsf(v[c]);
                if (a > amax) amax = a;
            }
            float s32 = amax / 6.0f;
            int s8 = csa2o_e4m3_encode(s32);
            float sd = (float)csa2o_e4m3_value(s8);
            scales[r * (width / 16) + g] = (uint8_t)s8;
            for (int c = 0; c < 16; c += 2) {
                int lo = 0, hi = 0;
                if (sd != 0.0f) {
                    lo = csa2o_e2m1_encode(v[c] / sd);
                    hi = csa2o_e2m1_encode(v[c + 1] / sd);
                }
                codes[r * (width / 2) + 8 * g + c / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* a2: FP8 rows (indexer K and per-layer SWA window).  The SWA window stays
 * FP8 (study notes section 4; myzaker "cache precision"); the indexer K is
 * FP8 E4M3 with one fp32 scale per token.
 * Reading: sigma = amax / 448 (fp32), code_c = E4M3_RNE_sat(x_c / sigma);
 * a zero sigma stores codes 0x00. */
EXPORT void csa2o_quantize_fp8(const uint16_t *x, int64_t rows, int width,
                               uint8_t *codes, float *scale) {
    e4m3_tab_init();
#pragma omp parallel for schedule(static) if (rows > 256)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * width;
        float amax = 0.0f;
        for (int c = 0; c < width; ++c) {
            float a = fabsf(csa2o_bf16_to_f32(xr[c]));
            if (a > amax) amax = a;
        }
        float sigma = amax / 448.0f;
        scale[r] = sigma;
        for (int c = 0; c < width; ++c) {
            int code = 0;
            if (sigma != 0.0f) code = csa2o_e4m3_encode(csa2o_bf16_to_f32(xr[c]) / sigma);
            codes[r * width + c] = (uint8_t)code;
        }
    }
}

/* Dequantise on read (study notes section 4: the cache is read back and
 * dequantised for attention).  Exact in fp64. */
EXPORT void csa2o_dequant_fp4(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                              int width, double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < width; ++c) {
            uint8_t byte = codes[r * (width / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 15);
            double s = csa2o_e4m3_value(scales[r * (width / 16) + c / 16]);
            out[r * width + c] = csa2o_e2m1_value(code) * s;
        }
}

EXPORT void csa2o_dequant_fp8(const uint8_t *codes, const float *scale, int64_t rows,
                              int width, double *out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < width; ++c)
            out[r * width + c] = csa2o_e4m3_value(codes[r * width + c]) * (double)scale[r];
}

/* ------------------------------------------------------------------------ */
/* RoPE inside the append                                                    */
/* ------------------------------------------------------------------------ */
/* The main KV is quantised after RoPE (myzaker "cache precision and tiering").
 * The pages give neither the rotated channels nor the angles, so both are
 * inputs: cs [n_pos][pairs][2] holds (cos, sin) of pair i at token position p;
 * pair i is channels start + 2i, start + 2i + 1 of a width-channel bf16 row.
 * Reading fixed for this build: a pair (x0, x1) becomes, in fp32 with the
 * products rounded first, y0 = fma(x0, c, -(x1 s)) and y1 = fma(x0, s, x1 c),
 * each rounded to bf16 -- the rows a separate RoPE step would store before the
 * append.  Other channels are copied.  pos[r] is row r's token position; a row
 * whose position is outside [0, n_pos) is copied unrotated.  Returns the number
 * of such rows. */
EXPORT int64_t csa2o_rope_rows(const uint16_t *x, int64_t rows, int width, const int64_t *pos,
                               const float *cs, int64_t n_pos, int start, int pairs,
                               uint16_t *out) {
    int64_t outside = 0;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * width;
        uint16_t *yr = out + r * width;
        memcpy(yr, xr, sizeof(uint16_t) * (size_t)width);
        int64_t p = pos[r];
        if (p < 0 || p >= n_pos) {
            ++outside;
            continue;
        }
        for (int i = 0; i < pairs; ++i) {
            int j = start + 2 * i;
            float x0 = csa2o_bf16_to_f32(xr[j]), x1 = csa2o_bf16_to_f32(xr[j + 1]);
            float c = cs[(p * pairs + i) * 2], sn = cs[(p * pairs + i) * 2 + 1];
            float m0 = x1 * sn;
            float m1 = x1 * c;
            yr[j] = csa2o_f32_to_bf16(fmaf(x0, c, -m0));
            yr[j + 1] = csa2o_f32_to_bf16(fmaf(x0, sn, m1));
        }
    }
    return outside;
}

/* ------------------------------------------------------------------------ */
/* Visibility                                                                */
/* ------------------------------------------------------------------------ */
/* The first Full layer scans every causally visible position (study notes
 * section 2; myzaker CSA2).  Encoder groups merge 2 tokens into 1 entry,
 * the decoder keeps ratio 1 (study notes section 3).  Reading: entry j covers
 * tokens [ratio*j, ratio*j + ratio) and is visible to the token at position t
 * once all of them are seen, so the visible entries are 0 .. (t+1)/ratio - 1. */
EXPORT int64_t csa2o_visible(int64_t t, int ratio) {
    if (t < 0) return 0;
    return (t + 1) / ratio;
}

/* ------------------------------------------------------------------------ */
/* a3: index score                                                           */
/* ------------------------------------------------------------------------ */
/* Limits of this plain implementation: H_I <= 16 index heads, d <= 256. */
/* score(s) = sum_h w_h * relu(q_h . k_s), k_s the dequantised FP8 indexer K
 * (the indexer K is projected from the main KV entry, myzaker CSA2).
 * The fp32 evaluation order is part of the definition, because it decides
 * Top-K membership:
 *   for each head h:  e = fmaf chain over even channels 0,2,4,..  (from +0)
 *                     o = fmaf chain over odd channels 1,3,5,..   (from +0)
 *                     a_h = e + o
 *   t = fmaf chain over h = 0..H_I-1 of (w_h, max(a_h, +0))     (from +0)
 *   score = t * sigma_s
 * k values enter as their exact E4M3 values (the per-token sigma is applied
 * once, at the end; relu commutes with the non-negative sigma).
 * kc: [.][d] codes, ks: [.] sigma; pos: positions to score (n of them);
 * q: bf16 [H_I][d]; w: [H_I]; out: [n]. */
EXPORT void csa2o_scores(const uint8_t *kc, const float *ks, int d, const int32_t *pos,
                         int64_t n, const uint16_t *q, const float *w, int H_I, float *out) {
    float qf[16][256];
    float kval[256];
    e4m3_tab_init();
    for (int c = 0; c < 256; ++c) kval[c] = (float)E4M3_TAB[c];
    for (int h = 0; h < H_I; ++h)
        for (int c = 0; c < d; ++c) qf[h][c] = csa2o_bf16_to_f32(q[h * d + c]);
#pragma omp parallel for schedule(static) if (n > 65536)
    for (int64_t i = 0; i < n; ++i) {
        int64_t s = pos ? pos[i] : i;
        const uint8_t *row = kc + s * (int64_t)d;
        float t = 0.0f;
        for (int h = 0; h < H_I; ++h) {
            float e = 0.0f, o = 0.0f;
            for (int c = 0; c < d; c += 2) {
                e = fmaf(qf[h][c], kval[row[c]], e);
                o = fmaf(qf[h][c + 1], kval[row[c + 1]], o);
            }
            float a = e + o;
            float r = (a > 0.0f) ? a : 0.0f;
            t = fmaf(w[h], r, t);
        }
        out[i] = t * ks[s];
    }
}

/* The same score without fp32 rounding, for a scan that sums in another order
 * (the tensor-core scan of prefill chunks): every product q_hc * k_sc and the
 * sums over channels and heads in fp64, then times sigma_s.  A bf16 times an
 * E4M3 value has at most 12 significant bits, so the products are exact and the
 * fp64 sums lose at most d * 2^-53 of the magnitude below -- far under any fp32
 * rounding.  mag_out[i] = sigma_s * sum_h w_h * sum_c |q_hc * k_sc|: the
 * magnitude that bounds the rounding error of any fp32 evaluation order of the
 * score (each of the d + H_I + 1 roundings costs at most 2^-24 of it, relative,
 * for round-to-nearest).  Same arguments as csa2o_scores. */
EXPORT void csa2o_scores_f64(const uint8_t *kc, const float *ks, int d, const int32_t *pos,
                             int64_t n, const uint16_t *q, const float *w, int H_I,
                             double *out, double *mag_out) {
    double qf[16][256];
    e4m3_tab_init();
    for (int h = 0; h < H_I; ++h)
        for (int c = 0; c < d; ++c) qf[h][c] = (double)csa2o_bf16_to_f32(q[h * d + c]);
#pragma omp parallel for schedule(static) if (n > 65536)
    for (int64_t i = 0; i < n; ++i) {
        int64_t s = pos ? pos[i] : i;
        const uint8_t *row = kc + s * (int64_t)d;
        double t = 0.0, m = 0.0;
        for (int h = 0; h < H_I; ++h) {
            double a = 0.0, am = 0.0;
            for (int c = 0; c < d; ++c) {
                double pr = qf[h][c] * E4M3_TAB[row[c]];
                a += pr;
                am += fabs(pr);
            }
            t += (double)w[h] * (a > 0.0 ? a : 0.0);
            m += (double)w[h] * am;
        }
        out[i] = t * (double)ks[s];
        if (mag_out) mag_out[i] = m * (double)ks[s];
    }
}

/* Block key for the hierarchical pool: the maximum score over the visible
 * positions of block b = [8b, 8b+8) (blocks of 8 positions, study notes
 * section 2 / report Figure 5; max over the block as fixed for this build). */
EXPORT void csa2o_block_max(const float *scores, int64_t N, float *bmax) {
    int64_t nb = (N + 7) / 8;
    for (int64_t b = 0; b < nb; ++b) {
        float m = -INFINITY;
        for (int64_t s = 8 * b; s < 8 * b + 8 && s < N; ++s)
            if (scores[s] > m) m = scores[s];
        bmax[b] = m;
    }
}

/* ------------------------------------------------------------------------ */
/* Selection: the first k items in the order (value descending, id ascending) */
/* ------------------------------------------------------------------------ */
/* Ties go to the lower index (fixed for this build); -0 equals +0 (plain
 * float comparison); NaN sorts after every number.  The result is returned
 * sorted by ascending id.  Plain full sort: O(n log n). */
typedef struct { float v; int32_t id; } vid_t;

static int cmp_value_desc(const void *pa, const void *pb) {
    const vid_t *a = (const vid_t *)pa, *b = (const vid_t *)pb;
    int an = isnan(a->v), bn = isnan(b->v);
    if (an != bn) return an ? 1 : -1;
    if (!an) {
        if (a->v > b->v) return -1;
        if (a->v < b->v) return 1;
    }
    return (a->id < b->id) ? -1 : (a->id > b->id);
}

static int cmp_i32(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

EXPORT int64_t csa2o_select_topk(const float *vals, const int32_t *ids, int64_t n, int64_t k,
                                 int32_t *out) {
    vid_t *t = (vid_t *)malloc(sizeof(vid_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) { t[i].v = vals[i]; t[i].id = ids ? ids[i] : (int32_t)i; }
    qsort(t, (size_t)n, sizeof(vid_t), cmp_value_desc);
    int64_t m = n < k ? n : k;
    for (int64_t i = 0; i < m; ++i) out[i] = t[i].id;
    qsort(out, (size_t)m, sizeof(int32_t), cmp_i32);
    free(t);
    return m;
}

/* ------------------------------------------------------------------------ */
/* a3-a5: Full layer for one query                                           */
/* ------------------------------------------------------------------------ */
/* The Full layer scans every visible position; in hierarchical mode it builds
 * the candidate pool from block scores, at most pool_blocks blocks x 8 =
 * 16384 positions (study notes section 2 / report Figure 5; myzaker CSA2), and
 * picks at most top_k <= 512 positions (study notes section 2).  Reading: the
 * Full layer's Top-K is taken over ALL visible positions ("scans all visible
 * positions"); flat mode (pool_blocks == 0) has no pool.
 * Outputs: pool_out [pool_blocks] ascending, -1 padded (may be NULL);
 * topk_out [top_k] ascending, -1 padded; scores_out [N] (may be NULL).
 * Returns the Top-K count. */
EXPORT int32_t csa2o_index_full_one(const uint8_t *kc, const float *ks, int d, int64_t N,
                                    const uint16_t *q, const float *w, int H_I,
                                    int pool_blocks, int top_k, int32_t *pool_out,
                                    int32_t *topk_out, float *scores_out) {
    float *sc = (float *)malloc(sizeof(float) * (size_t)(N > 0 ? N : 1));
    csa2o_scores(kc, ks, d, NULL, N, q, w, H_I, sc);
    if (pool_blocks > 0) {
        int64_t nb = (N + 7) / 8;
        float *bm = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
        int32_t *pl = (int32_t *)malloc(sizeof(int32_t) * (size_t)pool_blocks);
        csa2o_block_max(sc, N, bm);
        int64_t np = csa2o_select_topk(bm, NULL, nb, pool_blocks, pl);
        for (int64_t i = np; i < pool_blocks; ++i) pl[i] = -1;
        if (pool_out) memcpy(pool_out, pl, sizeof(int32_t) * (size_t)pool_blocks);
        free(pl);
        free(bm);
    }
    int64_t m = csa2o_select_topk(sc, NULL, N, top_k, topk_out);
    for (int64_t i = m; i < top_k; ++i) topk_out[i] = -1;
    if (scores_out) memcpy(scores_out, sc, sizeof(float) * (size_t)N);
    free(sc);
    return (int32_t)m;
}

/* a6: Reindex for one query.  A Reindex layer reuses the Full layer's global
 * KV and indexer K, re-scores with its own index query, and searches only
 * inside the pool (study notes section 2; myzaker CSA2).  Candidates: the
 * visible positions of the pool's blocks.  pool: [pool_blocks], -1 = unused. */
EXPORT int32_t csa2o_index_reindex_one(const uint8_t *kc, const float *ks, int d, int64_t N,
                                       const uint16_t *q, const float *w, int H_I,
                                       const int32_t *pool, int pool_blocks, int top_k,
                                       int32_t *topk_out) {
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * (size_t)(8 * pool_blocks + 1));
    int64_t n = 0;
    for (int i = 0; i < pool_blocks; ++i) {
        if (pool[i] < 0) continue;
        for (int64_t s = 8 * (int64_t)pool[i]; s < 8 * (int64_t)pool[i] + 8; ++s)
            if (s < N) cand[n++] = (int32_t)s;
    }
    float *sc = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    csa2o_scores(kc, ks, d, cand, n, q, w, H_I, sc);
    int64_t m = csa2o_select_topk(sc, cand, n, top_k, topk_out);
    for (int64_t i = m; i < top_k; ++i) topk_out[i] = -1;
    free(sc);
    free(cand);
    return (int32_t)m;
}

/* ------------------------------------------------------------------------ */
/* a8: sparse attention for one query                                        */
/* ------------------------------------------------------------------------ */
/* Each layer attends, with its own query, over the <= 512 selected global
 * entries (FP4, dequantised on read) together with its own 128-token FP8 SWA
 * window (study notes sections 1, 2, 4).  K = V = the 512-channel entry (MQA,
 * as fixed for this build).  Readings: one softmax over the union; the window
 * holds token positions max(0, t-swa_len+1) .. t, read from ring slot
 * pos % W; the two sets are not de-duplicated; logits are scaled by
 * softmax_scale; no sink.  fp64 throughout.
 * main_codes/main_scales: this request's rows [cap][256] / [cap][32];
 * swa_codes/swa_scale: this layer's ring [W][512] / [W]; q: bf16 [H][512];
 * topk: [top_k] entry ids (-1 = unused); out: [H][512]; lse: [H] (natural log;
 * -inf and o = 0 when there is no key). */
EXPORT void csa2o_attention_one(const uint8_t *main_codes, const uint8_t *main_scales,
                                const uint8_t *swa_codes, const float *swa_scale, int W,
                                const uint16_t *q, int H, int64_t t, const int32_t *topk,
                                int top_k, int swa_len, double softmax_scale, double *out,
                                double *lse) {
    const int D = 512;
    int64_t w0 = t - swa_len + 1;
    if (w0 < 0) w0 = 0;
    int nsel = 0;
    for (int i = 0; i < top_k; ++i) nsel += topk[i] >= 0;
    int64_t nkeys = nsel + (t - w0 + 1);
    if (swa_len <= 0) nkeys = nsel;
    double *kv = (double *)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1) * D);
    int64_t j = 0;
    for (int i = 0; i < top_k; ++i) {
        if (topk[i] < 0) continue;
        csa2o_dequant_fp4(main_codes + (int64_t)topk[i] * 256, main_scales + (int64_t)topk[i] * 32,
                          1, D, kv + j * D);
        ++j;
    }
    if (swa_len > 0)
        for (int64_t p = w0; p <= t; ++p) {
            int64_t slot = p % W;
            csa2o_dequant_fp8(swa_codes + slot * D, swa_scale + slot, 1, D, kv + j * D);
            ++j;
        }
    double *logit = (double *)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
    for (int h = 0; h < H; ++h) {
        double qh[512];
        for (int c = 0; c < D; ++c) qh[c] = (double)csa2o_bf16_to_f32(q[h * D + c]);
        double m = -INFINITY;
        for (int64_t k = 0; k < nkeys; ++k) {
            double s = 0.0;
            for (int c = 0; c < D; ++c) s += qh[c] * kv[k * D + c];
            logit[k] = s * softmax_scale;
            if (logit[k] > m) m = logit[k];
        }
        double *o = out + (int64_t)h * D;
        for (int c = 0; c < D; ++c) o[c] = 0.0;
        if (nkeys == 0) { lse[h] = -INFINITY; continue; }
        double den = 0.0;
        for (int64_t k = 0; k < nkeys; ++k) den += exp(logit[k] - m);
        for (int64_t k = 0; k < nkeys; ++k) {
            double p = exp(logit[k] - m) / den;
            for (int c = 0; c < D; ++c) o[c] += p * kv[k * D + c];
        }
        lse[h] = m + log(den);
    }
    free(logit);
    free(kv);
}

/* ------------------------------------------------------------------------ */
/* Batched drivers in the library's memory layout (OpenMP over queries)      */
/* ------------------------------------------------------------------------ */
/* Global KV of one group: main codes [B][cap][256], main scales [B][cap][32],
 * index codes [B][cap][d], index scales [B][cap].  Queries: [B][Tq][...]. */
EXPORT void csa2o_index_full(const uint8_t *kc, const float *ks, int B, int64_t cap, int d,
                             int ratio, const uint16_t *q, const float *w, const int32_t *q_pos,
                             int Tq, int H_I, int pool_blocks, int top_k, int32_t *pool_out,
                             int32_t *topk_out, int32_t *count_out) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < (int64_t)B * Tq; ++i) {
        int64_t b = i / Tq;
        int64_t N = csa2o_visible(q_pos[i], ratio);
        if (N > cap) N = cap;
        count_out[i] = csa2o_index_full_one(
            kc + b * cap * d, ks + b * cap, d, N, q + i * H_I * d, w + i * H_I, H_I,
            pool_blocks, top_k, pool_out ? pool_out + i * pool_blocks : NULL,
            topk_out + i * top_k, NULL);
    }
}

EXPORT void csa2o_index_reindex(const uint8_t *kc, const float *ks, int B, int64_t cap, int d,
                                int ratio, const uint16_t *q, const float *w,
                                const int32_t *q_pos, int Tq, int H_I, const int32_t *pool,
                                int pool_blocks, int top_k, int32_t *topk_out,
                                int32_t *count_out) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < (int64_t)B * Tq; ++i) {
        int64_t b = i / Tq;
        int64_t N = csa2o_visible(q_pos[i], ratio);
        if (N > cap) N = cap;
        count_out[i] = csa2o_index_reindex_one(kc + b * cap * d, ks + b * cap, d, N,
                                               q + i * H_I * d, w + i * H_I, H_I,
                                               pool + i * pool_blocks, pool_blocks, top_k,
                                               topk_out + i * top_k);
    }
}

EXPORT void csa2o_attention(const uint8_t *main_codes, const uint8_t *main_scales, int B,
                            int64_t cap, const uint8_t *swa_codes, const float *swa_scale, int W,
                            const uint16_t *q, const int32_t *q_pos, int Tq, int H,
                            const int32_t *topk, int top_k, int swa_len, double softmax_scale,
                            double *out, double *lse) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < (int64_t)B * Tq; ++i) {
        int64_t b = i / Tq;
        csa2o_attention_one(main_codes + b * cap * 256, main_scales + b * cap * 32,
                            swa_codes + b * (int64_t)W * 512, swa_scale + b * (int64_t)W, W,
                            q + i * (int64_t)H * 512, H, q_pos[i], topk + i * top_k, top_k,
                            swa_len, softmax_scale, out + i * (int64_t)H * 512, lse + i * H);
    }
}

/* Threads OpenMP will use (reported next to the CPU baseline). */
EXPORT int csa2o_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
