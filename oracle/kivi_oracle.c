/*
 * kivi_oracle.c -- slow, plain CPU oracle for the KIVI asymmetric 2-bit KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file; only the test-suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no source, header, table or helper with the
 * CUDA library under bit_asymmetric_kv_prefill_b200/csrc.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no FMA contraction anywhere, so every fp32 operation below rounds once, in
 * the order written).
 *
 * What it computes, and where the pages say so:
 *   - Keys are quantized per channel (min/max over G consecutive tokens of one
 *     channel) and values per token (min/max over G consecutive channels of one
 *     token), at 2 bits with group size 32:
 *       "KIVI Quantization Secures Llama-2 Accuracy at Two Bits" (paragraphs 1-3);
 *       record kv-efficiency/kivi-2bit-llama2-13b-mha-4k, fields "KV bytes basis"
 *       and "Quant method" (kivi-2bit-per-channel-k-per-token-v).
 *   - The code is asymmetric ("KIVI: A Tuning-Free Asymmetric 2bit Quantization
 *     for KV Cache", Key points).  The pages do not print the formula; this file
 *     takes the plain min/max reading: zero = group minimum, scale =
 *     (max - min)/3, code = clamp(rint((x - zero)/scale), 0, 3), with scale and
 *     zero stored as IEEE fp16 and the codes computed against the stored
 *     (rounded) scale and zero.
 *   - The newest R tokens stay in full precision and only grouped history is
 *     quantized (record field "KV bytes basis"; residual R = 128 in the
 *     "Methodology" field; the 128-token full-precision buffer in paragraph 4
 *     of the KIVI article).  Prefill of T tokens keeps
 *     n_q = R*floor((T-1)/R) quantized tokens and r = T - n_q in [1, R]
 *     residual tokens; an append into a full residual first quantizes all R
 *     residual tokens as tokens [n_q, n_q+R).
 *   - Keys may be quantized before RoPE and rotated after dequantization
 *     (KIVI article, paragraph 4; KVQuant summary, "Pre-RoPE Key Quantization").
 *     Rotate-half convention, absolute positions from 0, angle = fp32 product
 *     t * inv_freq_i with inv_freq_i = fp32(theta^(-2i/D)), cos/sin in double.
 *   - Decode attention is exact softmax attention of one query per head over
 *     the dequantized cache plus the residual, scale 1/sqrt(D), no mask, in
 *     double precision, stored as fp32.  Query head h reads KV head
 *     h / (H_q/H_kv).
 *
 * Every function works on ONE (batch, kv-head) sequence; callers loop.
 * Canonical (unpacked) layouts, all row-major:
 *   codesK [Tcap][D] uint8      sK, zK [Tcap/G][D] fp16 bits
 *   codesV [Tcap][D] uint8      sV, zV [Tcap][D/G] fp16 bits
 *   resK, resV [R][D] cache dtype bits (0 = fp16, 1 = bf16)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---- scalar conversions ------------------------------------------------- */

/* bfloat16 is the top half of an IEEE binary32. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE binary16 via the compiler's _Float16 (exact widening). */
static float f16_bits_to_float(uint16_t b)
{
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (float)h;
}

/* IEEE binary32 -> binary16, round to nearest even (compiler conversion). */
static uint16_t float_to_f16_bits(float f)
{
    _Float16 h = (_Float16)f;
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

static float load_elem(const uint16_t *p, long long i, int dtype)
{
    return dtype == 1 ? bf16_bits_to_float(p[i]) : f16_bits_to_float(p[i]);
}

float oracle_bf16_to_float(uint16_t b) { return bf16_bits_to_float(b); }
float oracle_f16_to_float(uint16_t b) { return f16_bits_to_float(b); }
uint16_t oracle_float_to_f16(float f) { return float_to_f16_bits(f); }

/* ---- residual split ------------------------------------------------------ */

/* Prefill split: n_q = R*floor((T-1)/R) quantized, r = T - n_q in [1, R]. */
void oracle_split(long long T, int R, long long *n_q, int *r)
{
    long long q = T >= 1 ? R * ((T - 1) / R) : 0;
    *n_q = q;
    *r = (int)(T - q);
}

/* ---- the 2-bit asymmetric group code ------------------------------------ */

/*
 * Quantize n values (already widened to fp32) sharing one scale and zero.
 * mn, mx: group min and max in fp32; s = fp16((mx - mn) / 3) with the
 * subtraction and division each rounded in fp32; z = fp16(mn); a stored zero
 * of either sign is written as +0.  If the stored scale is 0 every code is 0;
 * otherwise code = clamp(rint((x - z) / s), 0, 3) with the subtraction and
 * division in fp32 and rint rounding half to even.
 */
void oracle_quant_group(const float *x, int n, uint8_t *codes, uint16_t *s_bits,
                        uint16_t *z_bits)
{
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    float range = mx - mn;
    float s32 = range / 3.0f;
    uint16_t sb = float_to_f16_bits(s32);
    uint16_t zb = float_to_f16_bits(mn);
    if ((sb & 0x7fffu) == 0) sb = 0; /* -0 -> +0 */
    if ((zb & 0x7fffu) == 0) zb = 0;
    float sf = f16_bits_to_float(sb);
    float zf = f16_bits_to_float(zb);
    for (int i = 0; i < n; ++i) {
        int c = 0;
        if (sf != 0.0f) {
            float d = x[i] - zf;
            float y = d / sf;
            float rr = rintf(y);
            if (rr < 0.0f) rr = 0.0f;
            if (rr > 3.0f) rr = 3.0f;
            c = (int)rr;
        }
        codes[i] = (uint8_t)c;
    }
    *s_bits = sb;
    *z_bits = zb;
}

/* Keys, per channel: group g covers tokens [gG, gG+G) of every channel d.
 * src: rows [G][D] of the cache dtype (row stride D).  Writes codes rows
 * [G][D] (row stride D) and sK[d], zK[d] for d < D. */
void oracle_quant_k_group(const uint16_t *src, int D, int G, int dtype,
                          uint8_t *codes, uint16_t *sK, uint16_t *zK)
{
    float x[1024];
    uint8_t c[1024];
    for (int d = 0; d < D; ++d) {
        for (int t = 0; t < G; ++t) x[t] = load_elem(src, (long long)t * D + d, dtype);
        oracle_quant_group(x, G, c, &sK[d], &zK[d]);
        for (int t = 0; t < G; ++t) codes[(long long)t * D + d] = c[t];
    }
}

/* Values, per token: group j covers channels [jG, jG+G) of one token.
 * src: one row [D]; writes codes[D], sV[D/G], zV[D/G]. */
void oracle_quant_v_token(const uint16_t *src, int D, int G, int dtype,
                          uint8_t *codes, uint16_t *sV, uint16_t *zV)
{
    float x[1024];
    for (int j = 0; j < D / G; ++j) {
        for (int i = 0; i < G; ++i) x[i] = load_elem(src, (long long)j * G + i, dtype);
        oracle_quant_group(x, G, codes + (long long)j * G, &sV[j], &zV[j]);
    }
}

/* Quantize tokens [t0, t0+count) taken from rows src[count][D] (K and V) into
 * the canonical store; count is a multiple of G and t0 a multiple of G. */
static void quant_rows(const uint16_t *srcK, const uint16_t *srcV, long long t0,
                       long long count, int D, int G, int dtype, uint8_t *cK,
                       uint16_t *sK, uint16_t *zK, uint8_t *cV, uint16_t *sV,
                       uint16_t *zV)
{
    for (long long g = 0; g < count / G; ++g) {
        long long tg = t0 + g * G;
        oracle_quant_k_group(srcK + g * G * D, D, G, dtype, cK + tg * D,
                             sK + (tg / G) * D, zK + (tg / G) * D);
    }
    for (long long t = 0; t < count; ++t) {
        long long tt = t0 + t;
        oracle_quant_v_token(srcV + t * D, D, G, dtype, cV + tt * D,
                             sV + tt * (D / G), zV + tt * (D / G));
    }
}

/* Prefill one sequence with K, V rows [T][D]. */
void oracle_prefill_seq(const uint16_t *K, const uint16_t *V, long long T, int D,
                        int G, int R, int dtype, uint8_t *cK, uint16_t *sK,
                        uint16_t *zK, uint8_t *cV, uint16_t *sV, uint16_t *zV,
                        uint16_t *resK, uint16_t *resV, long long *n_q, int *r)
{
    long long nq;
    int rr;
    oracle_split(T, R, &nq, &rr);
    quant_rows(K, V, 0, nq, D, G, dtype, cK, sK, zK, cV, sV, zV);
    memcpy(resK, K + nq * D, (size_t)rr * D * sizeof(uint16_t));
    memcpy(resV, V + nq * D, (size_t)rr * D * sizeof(uint16_t));
    *n_q = nq;
    *r = rr;
}

/* Append one token (k, v rows [D]) to one sequence; flush a full residual. */
void oracle_append_seq(const uint16_t *k, const uint16_t *v, int D, int G, int R,
                       int dtype, uint8_t *cK, uint16_t *sK, uint16_t *zK,
                       uint8_t *cV, uint16_t *sV, uint16_t *zV, uint16_t *resK,
                       uint16_t *resV, long long *n_q, int *r)
{
    if (*r == R) {
        quant_rows(resK, resV, *n_q, R, D, G, dtype, cK, sK, zK, cV, sV, zV);
        *n_q += R;
        *r = 0;
    }
    memcpy(resK + (long long)(*r) * D, k, (size_t)D * sizeof(uint16_t));
    memcpy(resV + (long long)(*r) * D, v, (size_t)D * sizeof(uint16_t));
    *r += 1;
}

/* ---- dequantization, RoPE, attention ------------------------------------ */

/* Dequantized key row t (pre-rotation), in double: c*s + z is exact there. */
static void dequant_k_row(long long t, int D, int G, const uint8_t *cK,
                          const uint16_t *sK, const uint16_t *zK, double *out)
{
    for (int d = 0; d < D; ++d) {
        double s = f16_bits_to_float(sK[(t / G) * D + d]);
        double z = f16_bits_to_float(zK[(t / G) * D + d]);
        out[d] = (double)cK[t * D + d] * s + z;
    }
}

static void dequant_v_row(long long t, int D, int G, const uint8_t *cV,
                          const uint16_t *sV, const uint16_t *zV, double *out)
{
    for (int d = 0; d < D; ++d) {
        double s = f16_bits_to_float(sV[t * (D / G) + d / G]);
        double z = f16_bits_to_float(zV[t * (D / G) + d / G]);
        out[d] = (double)cV[t * D + d] * s + z;
    }
}

/* inv_freq_i = fp32(theta^(-2i/D)), i < D/2. */
void oracle_rope_inv_freq(int D, double theta, float *inv_freq)
{
    for (int i = 0; i < D / 2; ++i)
        inv_freq[i] = (float)pow(theta, -2.0 * (double)i / (double)D);
}

/* Rotate-half RoPE of row x at absolute position pos, in place.
 * Pair (i, i + D/2) with angle a = fp32(pos * inv_freq_i):
 *   x_i' = x_i cos a - x_{i+D/2} sin a,  x_{i+D/2}' = x_{i+D/2} cos a + x_i sin a. */
void oracle_rope_row(double *x, int D, long long pos, const float *inv_freq)
{
    for (int i = 0; i < D / 2; ++i) {
        float a = (float)pos * inv_freq[i];
        double c = cos((double)a), s = sin((double)a);
        double lo = x[i], hi = x[i + D / 2];
        x[i] = lo * c - hi * s;
        x[i + D / 2] = hi * c + lo * s;
    }
}

/*
 * Decode attention of HG query heads (q rows [HG][D], cache dtype) that share
 * this sequence's KV head.  out: [HG][D] fp32.  Scores q.k/sqrt(D) over the
 * n_q quantized tokens then the r residual tokens; softmax and the weighted
 * sum in double.
 */
void oracle_decode_seq(const uint16_t *q, int HG, int D, int G, int R, int dtype,
                       int pre_rope, double theta, const uint8_t *cK,
                       const uint16_t *sK, const uint16_t *zK, const uint8_t *cV,
                       const uint16_t *sV, const uint16_t *zV,
                       const uint16_t *resK, const uint16_t *resV, long long n_q,
                       int r, double *scores, float *out)
{
    (void)R;
    long long T = n_q + r;
    double krow[1024], vrow[1024], qd[1024], acc[1024];
    float inv_freq[512];
    if (pre_rope) oracle_rope_inv_freq(D, theta, inv_freq);
    double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (int h = 0; h < HG; ++h) {
        for (int d = 0; d < D; ++d) qd[d] = load_elem(q, (long long)h * D + d, dtype);
        double m = -INFINITY;
        for (long long t = 0; t < T; ++t) {
            if (t < n_q) {
                dequant_k_row(t, D, G, cK, sK, zK, krow);
            } else {
                for (int d = 0; d < D; ++d)
                    krow[d] = load_elem(resK, (t - n_q) * D + d, dtype);
            }
            if (pre_rope) oracle_rope_row(krow, D, t, inv_freq);
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += qd[d] * krow[d];
            s *= inv_sqrt_d;
            scores[t] = s;
            if (s > m) m = s;
        }
        double l = 0.0;
        for (int d = 0; d < D; ++d) acc[d] = 0.0;
        for (long long t = 0; t < T; ++t) {
            double p = exp(scores[t] - m);
            l += p;
            if (t < n_q) {
                dequant_v_row(t, D, G, cV, sV, zV, vrow);
            } else {
                for (int d = 0; d < D; ++d)
                    vrow[d] = load_elem(resV, (t - n_q) * D + d, dtype);
            }
            for (int d = 0; d < D; ++d) acc[d] += p * vrow[d];
        }
        for (int d = 0; d < D; ++d) out[(long long)h * D + d] = (float)(acc[d] / l);
    }
}

/* ---- diagnostic grouping modes (fake quantization) ----------------------- */

/*
 * The KIVI article (paragraphs 1-3) argues by comparing groupings: keys grouped
 * per token against per channel, values per channel against per token, and the
 * record for Llama-2-13B contrasts a naive symmetric 2-bit per-token scheme.
 * These functions quantize a whole [T][D] matrix under any of those groupings
 * and return the dequantized matrix, so that errors can be compared.
 *
 * One group of n values x_0..x_{n-1} (fp32), at `bits` bits:
 *   asymmetric (sym = 0), L = 2^bits - 1 levels above the zero:
 *     zero  = fp16(min), scale = fp16(fl32(fl32(max - min) / L)), a stored zero
 *             of either sign written as +0 (the KIVI code at bits = 2);
 *     code  = 0 if scale == 0, else clamp(rint(fl32(fl32(x - zero)/scale)), 0, L);
 *     x_hat = code*scale + zero rounded once to fp32.
 *   symmetric (sym = 1), L = 2^(bits-1) - 1, bits >= 2 (the plain absmax reading
 *   of "symmetric": no zero point, scale from the largest magnitude):
 *     scale = fp16(fl32(max|x| / L));
 *     code  = 0 if scale == 0, else clamp(rint(fl32(x/scale)), -(L+1), L);
 *     x_hat = code*scale (exact in fp32).
 * With outlier = 1 the group is split dense-and-sparse (KVQuant summary,
 * "Per-Vector Dense-and-Sparse Quantization"): its element of largest |x| (the
 * first one on ties) is kept exactly, x_hat = x, reported with code
 * FQ_OUTLIER_CODE, and the other n - 1 elements are quantized as above with the
 * statistics (min, max or max|x|) taken over them alone.
 * Codes are returned as int (may be NULL).
 */
#define FQ_OUTLIER_CODE (-1000)

static void fq_group(const float *x, long long stride, int n, int bits, int sym, int outlier,
                     float *xhat, int *codes)
{
    int o = -1; /* the sparse element, if any */
    if (outlier) {
        o = 0;
        for (int i = 1; i < n; ++i)
            if (fabsf(x[(long long)i * stride]) > fabsf(x[(long long)o * stride])) o = i;
        xhat[(long long)o * stride] = x[(long long)o * stride];
        if (codes) codes[(long long)o * stride] = FQ_OUTLIER_CODE;
        if (n == 1) return;
    }
    int first = o == 0 ? 1 : 0; /* first dense element */
    if (!sym) {
        float mn = x[(long long)first * stride], mx = mn;
        for (int i = first + 1; i < n; ++i) {
            if (i == o) continue;
            float v = x[(long long)i * stride];
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        int L = (1 << bits) - 1;
        uint16_t sb = float_to_f16_bits((mx - mn) / (float)L);
        uint16_t zb = float_to_f16_bits(mn);
        if ((sb & 0x7fffu) == 0) sb = 0;
        if ((zb & 0x7fffu) == 0) zb = 0;
        float sf = f16_bits_to_float(sb), zf = f16_bits_to_float(zb);
        for (int i = 0; i < n; ++i) {
            if (i == o) continue;
            long long at = (long long)i * stride;
            int c = 0;
            if (sf != 0.0f) {
                float rr = rintf((x[at] - zf) / sf);
                if (rr < 0.0f) rr = 0.0f;
                if (rr > (float)L) rr = (float)L;
                c = (int)rr;
            }
            xhat[at] = fmaf((float)c, sf, zf);
            if (codes) codes[at] = c;
        }
    } else {
        float amax = 0.0f;
        for (int i = 0; i < n; ++i) {
            if (i == o) continue;
            float a = fabsf(x[(long long)i * stride]);
            if (a > amax) amax = a;
        }
        int L = (1 << (bits - 1)) - 1;
        uint16_t sb = float_to_f16_bits(amax / (float)L);
        float sf = f16_bits_to_float(sb);
        for (int i = 0; i < n; ++i) {
            if (i == o) continue;
            long long at = (long long)i * stride;
            int c = 0;
            if (sf != 0.0f) {
                float rr = rintf(x[at] / sf);
                if (rr < (float)(-L - 1)) rr = (float)(-L - 1);
                if (rr > (float)L) rr = (float)L;
                c = (int)rr;
            }
            xhat[at] = (float)c * sf;
            if (codes) codes[at] = c;
        }
    }
}

/*
 * Fake-quantize one row-major [T][D] fp32 matrix.  axis 0 (per channel, the
 * KIVI key grouping): group g of channel d is tokens [gG, gG+G) of column d,
 * T a multiple of G.  axis 1 (per token, the KIVI value grouping): group j of
 * token t is channels [jG, jG+G) of row t, D a multiple of G.  outlier: 0 or 1
 * sparse elements per group.  Returns 0, or -1 for an unsupported argument.
 */
int oracle_fake_quant(const float *x, long long T, int D, int axis, int G, int bits,
                      int sym, int outlier, float *xhat, int *codes)
{
    if (G < 1 || bits < 1 || bits > 8 || (sym && bits < 2)) return -1;
    if (outlier != 0 && outlier != 1) return -1;
    if (axis == 0) {
        if (T % G) return -1;
        for (int d = 0; d < D; ++d)
            for (long long g = 0; g < T / G; ++g) {
                long long at = g * G * D + d;
                fq_group(x + at, D, G, bits, sym, outlier, xhat + at, codes ? codes + at : 0);
            }
        return 0;
    }
    if (axis == 1) {
        if (D % G) return -1;
        for (long long t = 0; t < T; ++t)
            for (int j = 0; j < D / G; ++j) {
                long long at = t * D + (long long)j * G;
                fq_group(x + at, 1, G, bits, sym, outlier, xhat + at, codes ? codes + at : 0);
            }
        return 0;
    }
    return -1;
}

/*
 * Non-uniform levels (KVQuant summary, "Non-Uniform KV Cache Quantization"; the
 * pages give only the name).  Each group keeps its min and max (fp32) and
 * codes every element by the nearest of nlev normalized levels 0 <= l_k <= 1
 * on [min, max]: u = (x - min)/(max - min) in double, code = argmin_k
 * |u - l_k| (the first level on ties), x_hat = fp32(min + (max - min) l_k).
 * A constant group decodes to its value with code 0.  Same axes as
 * oracle_fake_quant.  Returns 0, or -1 for an unsupported argument.
 */
static void cb_group(const float *x, long long stride, int n, int nlev, const double *lev,
                     float *xhat, int *codes)
{
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        float v = x[(long long)i * stride];
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    double range = (double)mx - (double)mn;
    for (int i = 0; i < n; ++i) {
        long long at = (long long)i * stride;
        int c = 0;
        if (range > 0.0) {
            double u = ((double)x[at] - (double)mn) / range;
            double best = fabs(u - lev[0]);
            for (int k = 1; k < nlev; ++k) {
                double e = fabs(u - lev[k]);
                if (e < best) {
                    best = e;
                    c = k;
                }
            }
            xhat[at] = (float)((double)mn + range * lev[c]);
        } else {
            xhat[at] = mn;
        }
        if (codes) codes[at] = c;
    }
}

int oracle_fake_quant_levels(const float *x, long long T, int D, int axis, int G, int nlev,
                             const double *levels, float *xhat, int *codes)
{
    if (G < 1 || nlev < 2 || nlev > 256) return -1;
    for (int k = 0; k < nlev; ++k)
        if (!(levels[k] >= 0.0 && levels[k] <= 1.0)) return -1;
    if (axis == 0) {
        if (T % G) return -1;
        for (int d = 0; d < D; ++d)
            for (long long g = 0; g < T / G; ++g) {
                long long at = g * G * D + d;
                cb_group(x + at, D, G, nlev, levels, xhat + at, codes ? codes + at : 0);
            }
        return 0;
    }
    if (axis == 1) {
        if (D % G) return -1;
        for (long long t = 0; t < T; ++t)
            for (int j = 0; j < D / G; ++j) {
                long long at = t * D + (long long)j * G;
                cb_group(x + at, 1, G, nlev, levels, xhat + at, codes ? codes + at : 0);
            }
        return 0;
    }
    return -1;
}

/* ---- byte accounting ----------------------------------------------------- */

/*
 * KV bytes per context token for a model of `layers` x `heads` x `head_dim`
 * (record kv-efficiency/kivi-2bit-llama2-13b-mha-4k, field "KV bytes basis"):
 *   grouped  = layers*heads*head_dim*2 (K and V)*bits/8 per token;
 *   residual = R*layers*heads*head_dim*2*dtype_bytes for the whole sequence,
 *              spread over `context` tokens;
 *   full     = layers*heads*head_dim*2*dtype_bytes per token (uncompressed).
 * Outputs: [0] grouped B/token, [1] residual B (total), [2] residual B/token,
 * [3] sum B/token, [4] full B/token, [5] full/sum ratio, [6] scale/zero
 * metadata B/token at fp16 scale and zero per group of G.
 */
void oracle_kv_bytes(long long layers, long long heads, long long head_dim,
                     long long R, long long context, int bits, int dtype_bytes,
                     long long G, double *out)
{
    double grouped = (double)(layers * heads * head_dim * 2) * bits / 8.0;
    double residual_total = (double)(R * layers * heads * head_dim * 2 * dtype_bytes);
    double residual_per_tok = residual_total / (double)context;
    double sum = grouped + residual_per_tok;
    double full = (double)(layers * heads * head_dim * 2 * dtype_bytes);
    /* K: one (scale, zero) pair per channel per G tokens; V: one pair per G
     * channels per token; each pair is 2 x fp16. */
    double meta = (double)(layers * heads) * 4.0 *
                  ((double)head_dim / (double)G + (double)head_dim / (double)G);
    out[0] = grouped;
    out[1] = residual_total;
    out[2] = residual_per_tok;
    out[3] = sum;
    out[4] = full;
    out[5] = full / sum;
    out[6] = meta;
}
