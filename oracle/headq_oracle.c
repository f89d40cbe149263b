/*
 * HeadQ CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of what HeadQ computes, used
 * only by the test-suite, the smoke check and the benchmark's CPU-baseline leg to
 * check the CUDA library.  Nothing in the product links or calls this file, and it
 * shares no code, header or table with the CUDA sources.
 *
 * Source: "HeadQ: Model-Visible Distortion and Score-Space Correction for KV-Cache
 * Quantization" -- the arXiv abstract (mlsanity.com / info.umar.mx records) and the
 * gist.science technical summary, whose section 3 ("Methodology: HeadQ",
 * algorithmic overview) gives the three steps calibrate / cache write / cache read,
 * and whose section 2 ("model-visible geometry") defines the score perturbation,
 * the Fisher-weighted KL surrogate, the readout error and the A^2 value weighting.
 *
 * Precision: the codec (base code, residual, side code) is emulated exactly in IEEE
 * fp32 -- compile with -ffp-contract=off and without fast-math so every operation
 * below is one correctly rounded fp32 operation and nothing is fused implicitly.
 * Attention and the diagnostics are computed in fp64 from the fp32 values.
 *
 * Readings of points the pages leave open (the same list is kept in the design
 * notes of the repository):
 *  - B_b, the "standard low-bit quantizer" of the base key, is per-token,
 *    group-of-32-channel (group = d when d < 32), asymmetric 2-bit min/max:
 *    scale = (max - min) / 3 (IEEE division), code = clamp(rint((x - min)/scale),
 *    0, 3) with round-half-even, all codes 0 when scale == 0; min and scale are
 *    stored as fp32; a -0 minimum or maximum is stored as +0.
 *  - Dequantisation is min + code*scale, the product rounded before the sum.
 *  - Q_q, the "low-bit side quantizer", is per-token 4-bit symmetric absmax:
 *    s = max|y| / 7, w = clamp(rint(y/s), -7, 7), all 0 when s == 0; w is stored
 *    as a 4-bit two's-complement nibble (even index in the low nibble), s as fp32.
 *  - The projection U_h^T e accumulates over channels c = 0..d-1 in order; each
 *    term U[c,i]*e_c is rounded to fp32 and then added with a second rounding
 *    (a plain multiply, then an add: no fused multiply-add).
 *  - Packing: channel c of the 2-bit code lives in byte c/4 at bit 2*(c%4).
 *  - An empty sequence (length 0) reads as output 0 and lse = -inf; all
 *    diagnostics are 0 for it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define HQO_API __attribute__((visibility("default")))

enum { HQO_OK = 0, HQO_BAD_ARG = 1, HQO_NO_MEM = 2 };

static int group_size(int d) { return d < 32 ? d : 32; }

static int shape_ok(int d, int r)
{
    if (d < 4 || d % 4 != 0) return 0;
    if (d >= 32 && d % 32 != 0) return 0;
    if (r < 0 || r > d || r % 2 != 0) return 0;
    return 1;
}

HQO_API int hqo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* Step 2a: the base low-bit key code k^base_j = B_b(k_j)                      */
/* (gist.science summary, section 3, cache write, first bullet).             */
/* ------------------------------------------------------------------------- */

static void base_quantize_token(const float *x, int d, uint8_t *packed,
                                float *scale, float *minimum)
{
    const int gs = group_size(d);
    memset(packed, 0, (size_t)d / 4);
    for (int g = 0; g * gs < d; ++g) {
        const float *xg = x + (size_t)g * gs;
        float lo = xg[0], hi = xg[0];
        for (int c = 1; c < gs; ++c) {
            if (xg[c] < lo) lo = xg[c];
            if (xg[c] > hi) hi = xg[c];
        }
        lo = lo + 0.0f; /* a -0 extreme becomes +0 */
        hi = hi + 0.0f;
        const float span = hi - lo;
        const float s = span / 3.0f;
        scale[g] = s;
        minimum[g] = lo;
        for (int c = 0; c < gs; ++c) {
            int code = 0;
            if (s != 0.0f) {
                const float off = xg[c] - lo;
                const float t = nearbyintf(off / s); /* default mode: half-even */
                code = t < 0.0f ? 0 : (t > 3.0f ? 3 : (int)t);
            }
            const int ch = g * gs + c;
            packed[ch >> 2] |= (uint8_t)(code << (2 * (ch & 3)));
        }
    }
}

static int code2_at(const uint8_t *packed, int c)
{
    return (packed[c >> 2] >> (2 * (c & 3))) & 3;
}

static void base_dequantize_token(const uint8_t *packed, const float *scale,
                                  const float *minimum, int d, float *xhat)
{
    const int gs = group_size(d);
    for (int c = 0; c < d; ++c) {
        const int g = c / gs;
        const float prod = (float)code2_at(packed, c) * scale[g];
        xhat[c] = minimum[g] + prod;
    }
}

/* The alternative base code (KIVI-style per-channel keys): for one block of  */
/* nt consecutive tokens x [nt, d] of one (b, kv), every channel c gets its  */
/* own minimum and scale over the block's tokens, with the same arithmetic as */
/* the per-token code (min/max, scale = (max - min)/3, rint half-even, clamp);*/
/* codes are packed per token exactly as in the per-token layout.            */
static void base_quantize_channel_block(const float *x, int nt, int d,
                                        uint8_t *packed, float *scale,
                                        float *minimum)
{
    memset(packed, 0, (size_t)nt * d / 4);
    for (int c = 0; c < d; ++c) {
        float lo = x[c], hi = x[c];
        for (int t = 1; t < nt; ++t) {
            const float v = x[(size_t)t * d + c];
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
        lo = lo + 0.0f;
        hi = hi + 0.0f;
        const float s = (hi - lo) / 3.0f;
        scale[c] = s;
        minimum[c] = lo;
        for (int t = 0; t < nt; ++t) {
            int code = 0;
            if (s != 0.0f) {
                const float tq = nearbyintf((x[(size_t)t * d + c] - lo) / s);
                code = tq < 0.0f ? 0 : (tq > 3.0f ? 3 : (int)tq);
            }
            packed[(size_t)t * (d / 4) + (c >> 2)] |= (uint8_t)(code << (2 * (c & 3)));
        }
    }
}

/* codes [seqs, T, d/4], scale/min [seqs, ceil(T/block), d] -> xhat [seqs, T, d] */
HQO_API int hqo_base_dequantize_channel(const uint8_t *codes, const float *scale,
                                        const float *minimum, int64_t seqs, int T,
                                        int d, int block, float *xhat)
{
    if (!shape_ok(d, 0) || seqs < 0 || T < 0 || block <= 0) return HQO_BAD_ARG;
    const int nblk = (T + block - 1) / block;
#pragma omp parallel for schedule(static)
    for (int64_t sq = 0; sq < seqs; ++sq)
        for (int t = 0; t < T; ++t) {
            const float *sc = scale + (sq * nblk + t / block) * d;
            const float *mn = minimum + (sq * nblk + t / block) * d;
            const uint8_t *pk = codes + (sq * T + t) * (d / 4);
            for (int c = 0; c < d; ++c) {
                const float prod = (float)code2_at(pk, c) * sc[c];
                xhat[(sq * T + t) * d + c] = mn[c] + prod;
            }
        }
    return HQO_OK;
}

HQO_API int hqo_base_dequantize(const uint8_t *codes, const float *scale,
                                const float *minimum, int64_t rows, int d,
                                float *xhat);

static void dequantize_keys(int kmode, int block, const uint8_t *kc, const float *ks,
                            const float *km, int64_t seqs, int T, int d, float *khat)
{
    if (kmode == 1)
        hqo_base_dequantize_channel(kc, ks, km, seqs, T, d, block, khat);
    else
        hqo_base_dequantize(kc, ks, km, seqs * T, d, khat);
}

/* x: [rows, d] -> codes [rows, d/4], scale/min [rows, ng] */
HQO_API int hqo_base_quantize(const float *x, int64_t rows, int d,
                              uint8_t *codes, float *scale, float *minimum)
{
    if (!shape_ok(d, 0) || rows < 0) return HQO_BAD_ARG;
    const int ng = d / group_size(d);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; ++t)
        base_quantize_token(x + t * d, d, codes + t * (d / 4), scale + t * ng,
                            minimum + t * ng);
    return HQO_OK;
}

HQO_API int hqo_base_dequantize(const uint8_t *codes, const float *scale,
                                const float *minimum, int64_t rows, int d,
                                float *xhat)
{
    if (!shape_ok(d, 0) || rows < 0) return HQO_BAD_ARG;
    const int ng = d / group_size(d);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; ++t)
        base_dequantize_token(codes + t * (d / 4), scale + t * ng,
                              minimum + t * ng, d, xhat + t * d);
    return HQO_OK;
}

/* ------------------------------------------------------------------------- */
/* Step 2b/2c: residual e_j = k_j - k^base_j, side code z_j = Q_q(U_h^T e_j)   */
/* (gist.science summary, section 3, cache write, second and third bullets). */
/* ------------------------------------------------------------------------- */

static void side_project(const float *e, const float *U, int d, int r, float *y)
{
    for (int i = 0; i < r; ++i) y[i] = 0.0f;
    for (int c = 0; c < d; ++c)
        for (int i = 0; i < r; ++i) {
            const float term = U[(size_t)c * r + i] * e[c]; /* rounded product */
            y[i] = y[i] + term;                              /* rounded sum */
        }
}

static void side_quantize(const float *y, int r, uint8_t *zc, float *zs)
{
    float a = 0.0f;
    for (int i = 0; i < r; ++i) {
        const float m = fabsf(y[i]);
        if (m > a) a = m;
    }
    const float s = a / 7.0f;
    memset(zc, 0, (size_t)r / 2);
    for (int i = 0; i < r; ++i) {
        int w = 0;
        if (s != 0.0f) {
            const float t = nearbyintf(y[i] / s);
            w = t < -7.0f ? -7 : (t > 7.0f ? 7 : (int)t);
        }
        zc[i >> 1] |= (uint8_t)((w & 0xF) << (4 * (i & 1)));
    }
    *zs = s;
}

static int nibble_at(const uint8_t *zc, int i)
{
    const int v = (zc[i >> 1] >> (4 * (i & 1))) & 0xF;
    return v >= 8 ? v - 16 : v;
}

/*
 * The whole cache write for keys: k [B, Hkv, n, d], U [Hkv, d, r].
 * Outputs kc [.., d/4], ks/km [.., ng], zc [.., r/2], zs [..]; y_out [.., r]
 * (nullable) receives the unquantised projection U_h^T e_j.
 */
HQO_API int hqo_cache_write(const float *k, int B, int Hkv, int n, int d, int r,
                            const float *U, uint8_t *kc, float *ks, float *km,
                            uint8_t *zc, float *zs, float *y_out, int kmode, int block)
{
    if (!shape_ok(d, r) || B < 0 || Hkv <= 0 || n < 0) return HQO_BAD_ARG;
    if (kmode != 0 && (kmode != 1 || block <= 0)) return HQO_BAD_ARG;
    const int ng = d / group_size(d);
    const int64_t rows = (int64_t)B * Hkv * n;
    if (kmode == 1) { /* per-channel base code over blocks of `block` tokens */
        const int nblk = (n + block - 1) / block;
#pragma omp parallel for schedule(static)
        for (int64_t sb = 0; sb < (int64_t)B * Hkv * nblk; ++sb) {
            const int64_t sq = sb / nblk;
            const int t0 = (int)(sb % nblk) * block;
            const int nt = n - t0 < block ? n - t0 : block;
            base_quantize_channel_block(k + (sq * n + t0) * d, nt, d,
                                        kc + (sq * n + t0) * (d / 4), ks + sb * d,
                                        km + sb * d);
        }
    }
    int bad = 0;
#pragma omp parallel
    {
        float *khat = malloc(sizeof(float) * (size_t)d);
        float *e = malloc(sizeof(float) * (size_t)d);
        float *y = malloc(sizeof(float) * (size_t)(r > 0 ? r : 1));
        if (!khat || !e || !y) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int64_t row = 0; row < rows; ++row) {
                const int kv = (int)((row / n) % Hkv);
                const float *x = k + row * d;
                uint8_t *codes = kc + row * (d / 4);
                if (kmode == 1) {
                    const int64_t sq = row / n;
                    const int t = (int)(row % n), nblk = (n + block - 1) / block;
                    const float *sc = ks + (sq * nblk + t / block) * d;
                    const float *mn = km + (sq * nblk + t / block) * d;
                    for (int c = 0; c < d; ++c) {
                        const float prod = (float)code2_at(codes, c) * sc[c];
                        khat[c] = mn[c] + prod;
                    }
                } else {
                    float *sc = ks + row * ng, *mn = km + row * ng;
                    base_quantize_token(x, d, codes, sc, mn);
                    base_dequantize_token(codes, sc, mn, d, khat);
                }
                for (int c = 0; c < d; ++c) e[c] = x[c] - khat[c];
                if (r > 0) {
                    side_project(e, U + (size_t)kv * d * r, d, r, y);
                    side_quantize(y, r, zc + row * (r / 2), zs + row);
                    if (y_out) memcpy(y_out + row * r, y, sizeof(float) * (size_t)r);
                } else {
                    zs[row] = 0.0f;
                }
            }
        }
        free(khat);
        free(e);
        free(y);
    }
    return bad ? HQO_NO_MEM : HQO_OK;
}

/* Q_q alone on given projections: y [rows, r] -> zc [rows, r/2], zs [rows] */
HQO_API int hqo_side_quantize(const float *y, int64_t rows, int r, uint8_t *zc,
                              float *zs)
{
    if (r < 0 || r % 2 || rows < 0) return HQO_BAD_ARG;
    for (int64_t t = 0; t < rows; ++t)
        side_quantize(y + t * r, r, zc + t * (r / 2), zs + t);
    return HQO_OK;
}

/* z^_j = w_j * s_j as fp32 (zc [rows, r/2], zs [rows] -> zhat [rows, r]) */
HQO_API int hqo_side_dequantize(const uint8_t *zc, const float *zs, int64_t rows,
                                int r, float *zhat)
{
    if (r < 0 || r % 2 || rows < 0) return HQO_BAD_ARG;
    for (int64_t t = 0; t < rows; ++t)
        for (int i = 0; i < r; ++i)
            zhat[t * r + i] = (float)nibble_at(zc + t * (r / 2), i) * zs[t];
    return HQO_OK;
}

/* ------------------------------------------------------------------------- */
/* Step 3: cache read.  s^_j = q^T k^base_j / sqrt(d) + q^T U_h z^_j / sqrt(d) */
/* (gist.science summary, section 3, cache read), then p = softmax(s^) and the */
/* attention-weighted readout o = sum_j p_j v_j (section 1 and 2.2).          */
/* sm_scale plays 1/sqrt(d); sigma multiplies the correction term (+1 is    */
/* HeadQ, 0 the base code alone, -1 the wrong-sign control of section 4).    */
/* ------------------------------------------------------------------------- */

static double dot_fd(const float *a, const float *b, int n)
{
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += (double)a[i] * (double)b[i];
    return s;
}

/* logits of one (query head, sequence) against T keys, fp64 */
static void headq_logits(const float *q, const float *khat, const double *zhat,
                         const float *U, int T, int d, int r, double sm_scale,
                         double sigma, double *s, double *uz)
{
    for (int j = 0; j < T; ++j) {
        double base = dot_fd(q, khat + (size_t)j * d, d);
        double corr = 0.0;
        if (zhat) {
            /* U_h z^_j, a d-vector, then its inner product with q */
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int i = 0; i < r; ++i)
                    acc += (double)U[(size_t)c * r + i] * zhat[(size_t)j * r + i];
                uz[c] = acc;
            }
            for (int c = 0; c < d; ++c) corr += (double)q[c] * uz[c];
        }
        s[j] = sm_scale * (base + sigma * corr);
    }
}

static double log_sum_exp(const double *s, int T)
{
    double m = -INFINITY;
    for (int j = 0; j < T; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int j = 0; j < T; ++j) l += exp(s[j] - m);
    return m + log(l);
}

/*
 * q [B, Hq, d]; khat, v [B, Hkv, T, d]; zhat [B, Hkv, T, r] (nullable: no
 * correction); U [Hkv, d, r].  Head h reads KV head h / (Hq/Hkv).  seq_lens [B]
 * nullable (all T).  out [B, Hq, d], lse [B, Hq], logits [B, Hq, T] (nullable).
 */
HQO_API int hqo_attend(const float *q, int B, int Hq, int Hkv, int T, int d, int r,
                       const int32_t *seq_lens, const float *khat,
                       const double *zhat, const float *U, const float *v,
                       double sm_scale, double sigma, double *out, double *lse,
                       double *logits)
{
    if (B < 0 || Hkv <= 0 || Hq % Hkv != 0 || T < 0 || d <= 0 || r < 0)
        return HQO_BAD_ARG;
    const int G = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double *s = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *uz = malloc(sizeof(double) * (size_t)d);
        if (!s || !uz) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(2) schedule(dynamic)
            for (int b = 0; b < B; ++b)
                for (int h = 0; h < Hq; ++h) {
                    const int kv = h / G;
                    const int Tb = seq_lens ? seq_lens[b] : T;
                    const size_t row = (size_t)b * Hkv + kv;
                    const float *qh = q + ((size_t)b * Hq + h) * d;
                    double *o = out + ((size_t)b * Hq + h) * d;
                    for (int c = 0; c < d; ++c) o[c] = 0.0;
                    if (Tb <= 0) {
                        lse[(size_t)b * Hq + h] = -INFINITY;
                        continue;
                    }
                    headq_logits(qh, khat + row * T * d,
                                 zhat ? zhat + row * T * r : NULL,
                                 U + (size_t)kv * d * r, Tb, d, r, sm_scale, sigma,
                                 s, uz);
                    const double L = log_sum_exp(s, Tb);
                    for (int j = 0; j < Tb; ++j) {
                        const double p = exp(s[j] - L);
                        const float *vj = v + (row * T + j) * d;
                        for (int c = 0; c < d; ++c) o[c] += p * (double)vj[c];
                    }
                    lse[(size_t)b * Hq + h] = L;
                    if (logits)
                        for (int j = 0; j < T; ++j)
                            logits[((size_t)b * Hq + h) * T + j] =
                                j < Tb ? s[j] : -INFINITY;
                }
        }
        free(s);
        free(uz);
    }
    return bad ? HQO_NO_MEM : HQO_OK;
}

/* Values as the cache read sees them: dense copy, or the 2-bit code dequantised. */
static int values_as_read(int vmode, const float *v_dense, const uint8_t *vc,
                          const float *vs, const float *vm, int64_t rows, int d,
                          float **v_out, int *owned)
{
    *owned = 0;
    if (vmode == 0) {
        *v_out = (float *)v_dense;
        return v_dense ? HQO_OK : HQO_BAD_ARG;
    }
    float *vv = malloc(sizeof(float) * (size_t)(rows * d > 0 ? rows * d : 1));
    if (!vv) return HQO_NO_MEM;
    hqo_base_dequantize(vc, vs, vm, rows, d, vv);
    *v_out = vv;
    *owned = 1;
    return HQO_OK;
}

/*
 * Cache read from the stored planes: dequantise the base key code and the side
 * code, then attend.  Planes are [B, Hkv, T, ...] with exactly T tokens.
 * vmode 0: v_dense [B,Hkv,T,d]; vmode 1: vc/vs/vm 2-bit planes.
 */
HQO_API int hqo_decode(const float *q, int B, int Hq, int Hkv, int T, int d, int r,
                       const int32_t *seq_lens, const uint8_t *kc, const float *ks,
                       const float *km, const uint8_t *zc, const float *zs,
                       const float *U, int vmode, const float *v_dense,
                       const uint8_t *vc, const float *vs, const float *vm,
                       double sm_scale, double sigma, double *out, double *lse,
                       int kmode, int block)
{
    if (!shape_ok(d, r)) return HQO_BAD_ARG;
    const int64_t rows = (int64_t)B * Hkv * T;
    float *khat = malloc(sizeof(float) * (size_t)(rows * d > 0 ? rows * d : 1));
    float *zf = malloc(sizeof(float) * (size_t)(rows * r > 0 ? rows * r : 1));
    double *zhat = malloc(sizeof(double) * (size_t)(rows * r > 0 ? rows * r : 1));
    float *vv = NULL;
    int owned = 0, rc = HQO_NO_MEM;
    if (khat && zf && zhat) {
        dequantize_keys(kmode, block, kc, ks, km, (int64_t)B * Hkv, T, d, khat);
        hqo_side_dequantize(zc, zs, rows, r, zf);
        for (int64_t i = 0; i < rows * r; ++i) zhat[i] = (double)zf[i];
        rc = values_as_read(vmode, v_dense, vc, vs, vm, rows, d, &vv, &owned);
        if (rc == HQO_OK)
            rc = hqo_attend(q, B, Hq, Hkv, T, d, r, seq_lens, khat, zhat, U, vv,
                            sm_scale, sigma, out, lse, NULL);
    }
    if (owned) free(vv);
    free(khat);
    free(zf);
    free(zhat);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Step 4: model-visible distortion diagnostics (gist.science summary,        */
/* section 2.1: delta s_j = q^T delta k_j / sqrt(d), KL of the attention      */
/* distributions, locally the Fisher-weighted variance of the score error;    */
/* section 2.2: readout error delta o = sum_j p_j delta v_j at fixed p and     */
/* the A^2 (p_j^2) weighted token distortion).  p is the full-precision       */
/* attention softmax(s), p~ the HeadQ one softmax(s^).                         */
/*   kl    = KL(p || p~) = sum_j p_j (s_j - s^_j) - lse(s) + lse(s^)          */
/*   fvar  = Var_p(s^ - s) = sum_j p_j d_j^2 - (sum_j p_j d_j)^2               */
/*   a2v   = sum_j p_j^2 |v^_j - v_j|^2                                        */
/*   dout2 = |sum_j p_j (v^_j - v_j)|^2                                        */
/* ------------------------------------------------------------------------- */

HQO_API int hqo_attn_kl(const float *q, int B, int Hq, int Hkv, int T, int d, int r,
                        const int32_t *seq_lens, const uint8_t *kc, const float *ks,
                        const float *km, const uint8_t *zc, const float *zs,
                        const float *U, int vmode, const float *v_dense,
                        const uint8_t *vc, const float *vs, const float *vm,
                        const float *k_full, const float *v_full, double sm_scale,
                        double sigma, double *kl, double *fvar, double *a2v,
                        double *dout2, int kmode, int block)
{
    if (!shape_ok(d, r) || Hkv <= 0 || Hq % Hkv) return HQO_BAD_ARG;
    const int G = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hkv * T;
    float *khat = malloc(sizeof(float) * (size_t)(rows * d > 0 ? rows * d : 1));
    float *zf = malloc(sizeof(float) * (size_t)(rows * r > 0 ? rows * r : 1));
    double *zhat = malloc(sizeof(double) * (size_t)(rows * r > 0 ? rows * r : 1));
    float *vv = NULL;
    int owned = 0, rc = HQO_NO_MEM;
    if (!khat || !zf || !zhat) goto done;
    dequantize_keys(kmode, block, kc, ks, km, (int64_t)B * Hkv, T, d, khat);
    hqo_side_dequantize(zc, zs, rows, r, zf);
    for (int64_t i = 0; i < rows * r; ++i) zhat[i] = (double)zf[i];
    rc = values_as_read(vmode, v_dense, vc, vs, vm, rows, d, &vv, &owned);
    if (rc != HQO_OK) goto done;
    int bad = 0;
#pragma omp parallel
    {
        double *s = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *sh = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *uz = malloc(sizeof(double) * (size_t)d);
        double *dov = malloc(sizeof(double) * (size_t)d);
        if (!s || !sh || !uz || !dov) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(2) schedule(dynamic)
            for (int b = 0; b < B; ++b)
                for (int h = 0; h < Hq; ++h) {
                    const int kv = h / G;
                    const int Tb = seq_lens ? seq_lens[b] : T;
                    const size_t row = (size_t)b * Hkv + kv, bh = (size_t)b * Hq + h;
                    const float *qh = q + bh * d;
                    kl[bh] = fvar[bh] = a2v[bh] = dout2[bh] = 0.0;
                    if (Tb <= 0) continue;
                    /* full-precision logits s_j and HeadQ logits s^_j */
                    headq_logits(qh, k_full + row * T * d, NULL, U, Tb, d, r,
                                 sm_scale, 0.0, s, uz);
                    headq_logits(qh, khat + row * T * d, zhat + row * T * r,
                                 U + (size_t)kv * d * r, Tb, d, r, sm_scale, sigma,
                                 sh, uz);
                    const double L = log_sum_exp(s, Tb), Lh = log_sum_exp(sh, Tb);
                    double e1 = 0.0, m1 = 0.0, m2 = 0.0, a2 = 0.0;
                    for (int c = 0; c < d; ++c) dov[c] = 0.0;
                    for (int j = 0; j < Tb; ++j) {
                        const double p = exp(s[j] - L);
                        const double dl = sh[j] - s[j];
                        e1 += p * (s[j] - sh[j]);
                        m1 += p * dl;
                        m2 += p * dl * dl;
                        const float *vj = vv + (row * T + j) * d;
                        const float *fj = v_full + (row * T + j) * d;
                        double n2 = 0.0;
                        for (int c = 0; c < d; ++c) {
                            const double dv = (double)vj[c] - (double)fj[c];
                            n2 += dv * dv;
                            dov[c] += p * dv;
                        }
                        a2 += p * p * n2;
                    }
                    double o2 = 0.0;
                    for (int c = 0; c < d; ++c) o2 += dov[c] * dov[c];
                    kl[bh] = e1 - L + Lh;
                    fvar[bh] = m2 - m1 * m1;
                    a2v[bh] = a2;
                    dout2[bh] = o2;
                }
        }
        free(s);
        free(sh);
        free(uz);
        free(dov);
    }
    rc = bad ? HQO_NO_MEM : HQO_OK;
done:
    if (owned) free(vv);
    free(khat);
    free(zf);
    free(zhat);
    return rc;
}
