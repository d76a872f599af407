/*
 * CSA2 reference oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of what the CSA2 hot path
 * computes.  Only the test-suite, the smoke check and the CPU-baseline and
 * reference legs of the benchmark may load it.  It shares no code, header, table or constant
 * generator with the CUDA library, and the library never calls it.
 *
 * Sources (web pages about the DeepSeek V4.1 Flash report):
 *   [A] "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径" (kongchang.com)
 *   [B] "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型" (ai.chattools.top)
 * Section names below are those pages' headings.
 *
 * Precision.  The pages fix the storage formats (E2M1 codes, one E4M3 scale
 * per 16 channels, an 8-bit sliding window).  Quantisers therefore round the
 * exact quotient once.  They divide in fp64, and that is enough.  Take a
 * rounding midpoint m of E2M1 or E4M3 (at most 5 significant bits) and fp32
 * operands a, b (24 bits).  If a != b*m, then a - b*m is a nonzero multiple of
 * the smaller of a's lowest significand bit and the product of b's and m's.
 * That step is at least about 2^-29 |b*m|, so |a/b - m| is at least about
 * 2^-29 |m|, while the fp64 quotient errs by at most 2^-53 |a/b|.  The fp64
 * quotient therefore lies on the same side of every midpoint as the exact
 * one, and equals a midpoint only when the exact quotient does.  Indexer scores are
 * fp32 in one fixed summation order, because an integer decision (the top-K
 * set) hangs on them and both sides must take it in the same precision.
 * Attention is computed in fp64.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* E2M1 (FP4): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
 * [B §FP4 量化 + Bounded Replay]: main KV is stored as E2M1.
 * Magnitudes of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Bit 3 is the sign. */
double oracle_e2m1_value(int code)
{
    int e = (code >> 1) & 3, m = code & 1;
    double mag;
    if (e == 0)
        mag = 0.5 * m;                       /* subnormal: m * 2^(1-1) * 0.5 */
    else
        mag = ldexp(1.0 + 0.5 * m, e - 1);   /* normal: 2^(e-1) * (1 + m/2) */
    return (code & 8) ? -mag : mag;
}

/* E4M3 (OCP "fn" variant): bias 7, no infinities, 0x7F/0xFF are NaN,
 * largest finite magnitude 448.  [B §FP4 量化 + Bounded Replay]: one E4M3
 * scale per 16 channels. */
double oracle_e4m3_value(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);              /* m/8 * 2^-6 */
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round |v| to E2M1 with round-to-nearest-even and saturation at 6.
 * The sign is kept even when the magnitude rounds to zero (-0 -> code 8).
 * Done by enumerating the eight representable magnitudes: pick the nearest,
 * on a tie the one whose mantissa bit is 0. */
int oracle_e2m1_encode(double v)
{
    int sign = signbit(v) ? 8 : 0;
    double a = fabs(v);
    if (a >= 6.0)
        return sign | 7;      /* saturate: at huge |v| the distances below round equal */
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double err = fabs(oracle_e2m1_value(c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return sign | best;
}

/* Round v to E4M3 with round-to-nearest-even; finite values beyond 448
 * saturate to 448 ("satfinite").  Sign kept for values that round to 0. */
int oracle_e4m3_encode(double v)
{
    int sign = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    int code;
    if (a >= 448.0) {
        code = 0x7E;                            /* 448 */
    } else if (a < ldexp(1.0, -6)) {
        /* subnormal range: value = m * 2^-9, m in 0..8 (m == 8 is 2^-6,
         * which is the smallest normal and has code 8: continuous). */
        double m = rint(ldexp(a, 9));            /* rint: ties to even */
        code = (int)m;
    } else {
        int e2;
        double fr = frexp(a, &e2);               /* a = fr * 2^e2, fr in [0.5,1) */
        int e = e2 - 1;                          /* a = (2fr) * 2^e, 2fr in [1,2) */
        double m = rint((2.0 * fr - 1.0) * 8.0); /* exact scaling, RNE */
        if (m == 8.0) { m = 0.0; e += 1; }
        code = ((e + 7) << 3) | (int)m;
        if (code > 0x7E) code = 0x7E;            /* satfinite */
    }
    return sign | code;
}

/* ------------------------------------------------------------------------ */
/* A1/A2: FP4 quantise-on-write.  [B §FP4 量化 + Bounded Replay]            */
/* Per block of 16 channels: s = E4M3(amax / 6); codes = E2M1(x / s).       */
/* No second-level (global) scale.  Two codes per byte, element 2i in the   */
/* low nibble.  A zero scale gives all-zero codes.                          */
/* ------------------------------------------------------------------------ */
void oracle_quantize_fp4(const float *x, int64_t rows, int dim,
                         uint8_t *codes, uint8_t *scales)
{
    int nblk = dim / 16;
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * dim;
        uint8_t *cr = codes + r * (dim / 2);
        uint8_t *sr = scales + r * nblk;
        for (int b = 0; b < nblk; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 16; ++i) {
                double a = fabs((double)xr[b * 16 + i]);
                if (a > amax) amax = a;
            }
            int sc = oracle_e4m3_encode(amax / 6.0);
            double s = oracle_e4m3_value(sc);
            sr[b] = (uint8_t)sc;
            for (int i = 0; i < 16; i += 2) {
                int c0 = 0, c1 = 0;
                if (s != 0.0) {
                    c0 = oracle_e2m1_encode((double)xr[b * 16 + i] / s);
                    c1 = oracle_e2m1_encode((double)xr[b * 16 + i + 1] / s);
                }
                cr[(b * 16 + i) / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Sequence compressor + quantise-on-write.  [B §CSA2：三层压缩一次吃满]:   */
/* every m tokens become one entry (V4's CSA compresses along the sequence; */
/* its weights are learned and not on the pages).  With caller-supplied     */
/* per-token weights w[e][i], entry e = sum_{i<m} w[e][i] * x[m e + i]:      */
/* fp32, tokens in order, each product and each sum rounded once (no fused  */
/* multiply-add).  w == NULL means the plain mean, w = 1/m.  The entry then */
/* goes through the FP4 quantiser above.                                    */
/* ------------------------------------------------------------------------ */
void oracle_compress_fp4(const float *x, int64_t entries, int ratio, int dim,
                         const float *w, uint8_t *codes, uint8_t *scales)
{
    float *row = (float *)malloc(sizeof(float) * (size_t)dim);
    const float mean_w = 1.0f / (float)ratio;
    for (int64_t e = 0; e < entries; ++e) {
        for (int c = 0; c < dim; ++c) {
            float acc = 0.0f;
            for (int i = 0; i < ratio; ++i) {
                const float wi = w ? w[e * ratio + i] : mean_w;
                const float prod = wi * x[(e * ratio + i) * (int64_t)dim + c];
                acc = (i == 0) ? prod : acc + prod;
            }
            row[c] = acc;
        }
        oracle_quantize_fp4(row, 1, dim, codes + e * (dim / 2), scales + e * (dim / 16));
    }
    free(row);
}

/* Dequantised FP4 value of channel c of one row (exact in fp64 and fp32). */
static double fp4_value(const uint8_t *codes, const uint8_t *scales, int c)
{
    int byte = codes[c >> 1];
    int code = (c & 1) ? (byte >> 4) : (byte & 15);
    return oracle_e2m1_value(code) * oracle_e4m3_value(scales[c >> 4]);
}

void oracle_dequantize_fp4(const uint8_t *codes, const uint8_t *scales,
                           int64_t rows, int dim, double *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < dim; ++c)
            out[r * dim + c] = fp4_value(codes + r * (dim / 2), scales + r * (dim / 16), c);
}

/* ------------------------------------------------------------------------ */
/* A3: sliding-window (SWA) write.  [A §压缩吸收注意力（二代）] keeps the     */
/* window at 8 bits; [B §FP4 量化 + Bounded Replay] truncates it to 128.    */
/* Reading: E4M3 codes with one fp32 scale per token, s = amax/448 rounded  */
/* to fp32; code = E4M3(x / s) rounded once from the exact quotient.        */
/* ------------------------------------------------------------------------ */
void oracle_quantize_fp8_token(const float *x, int64_t rows, int dim,
                               uint8_t *codes, float *scales)
{
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * dim;
        float amax = 0.0f;
        for (int i = 0; i < dim; ++i) {
            float a = fabsf(xr[i]);
            if (a > amax) amax = a;
        }
        float s = amax / 448.0f;                   /* fp32, round to nearest */
        scales[r] = s;
        for (int i = 0; i < dim; ++i)
            codes[r * dim + i] = (uint8_t)(s == 0.0f ? 0
                                   : oracle_e4m3_encode((double)xr[i] / (double)s));
    }
}

/* ------------------------------------------------------------------------ */
/* A4: indexer score of one query row against n keys.                       */
/* [B §为什么 KV 缓存成了新瓶颈] names DSA's indexer; reading: its form       */
/* I_j = sum_h w_h * ReLU(q_h . k_j), k shared by the heads.  Both q and k  */
/* are FP4 with E4M3/16 scales ([B §FP4 量化 + Bounded Replay]).            */
/* fp32 with a fixed order: per 16-channel block the partial sum is exact   */
/* (every term is a multiple of s_q*s_k/4 and the block total needs at most */
/* 20 significant bits), blocks are added left to right, heads are added    */
/* left to right as acc = acc + w_h * relu(dot_h), no fused multiply-add,   */
/* and a zero result is returned as +0.                                     */
/* q_codes: [H][32], q_scales: [H][4], w: [H], k rows via strides (bytes).  */
/* key_index: optional list of key rows to score (NULL = rows 0..n-1).      */
/* ------------------------------------------------------------------------ */
void oracle_index_scores(const uint8_t *q_codes, const uint8_t *q_scales,
                         const float *w, int H,
                         const uint8_t *k_codes, int64_t k_code_stride,
                         const uint8_t *k_scales, int64_t k_scale_stride,
                         const int32_t *key_index, int64_t n, float *scores)
{
    /* dequantised query, fp32 (exact) */
    float *qv = (float *)malloc(sizeof(float) * H * 64);
    for (int h = 0; h < H; ++h)
        for (int c = 0; c < 64; ++c)
            qv[h * 64 + c] = (float)fp4_value(q_codes + h * 32, q_scales + h * 4, c);

    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        int64_t row = key_index ? (int64_t)key_index[j] : j;
        const uint8_t *kc = k_codes + row * k_code_stride;
        const uint8_t *ks = k_scales + row * k_scale_stride;
        float kv[64];
        for (int c = 0; c < 64; ++c)
            kv[c] = (float)fp4_value(kc, ks, c);
        float acc = 0.0f;
        for (int h = 0; h < H; ++h) {
            float p[4];
            for (int b = 0; b < 4; ++b) {
                float s = 0.0f;
                for (int i = 0; i < 16; ++i) {
                    float prod = qv[h * 64 + b * 16 + i] * kv[b * 16 + i];
                    s = s + prod;
                }
                p[b] = s;
            }
            float dot = ((p[0] + p[1]) + p[2]) + p[3];
            float r = dot > 0.0f ? dot : 0.0f;
            float t = w[h] * r;
            acc = acc + t;
        }
        if (acc == 0.0f) acc = 0.0f;   /* -0 -> +0 */
        scores[j] = acc;
    }
    free(qv);
}

/* ------------------------------------------------------------------------ */
/* A5: top-K.  [A §压缩吸收注意力（二代）]: the indexer picks 2048 blocks.   */
/* Order: score descending, index ascending on ties.  A full sort; take the */
/* first min(K, n); return them in ascending index order, padded with -1.   */
/* ------------------------------------------------------------------------ */
typedef struct { float s; int32_t i; } scored_t;

static int cmp_desc(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x < y) ? -1 : (x > y);
}

/* scores[j] belongs to entry ids[j] (ids NULL = j).  Returns count. */
int32_t oracle_topk(const float *scores, const int32_t *ids, int64_t n,
                    int32_t K, int32_t *out_idx)
{
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (n > 0 ? n : 1));
    for (int64_t j = 0; j < n; ++j) {
        v[j].s = scores[j];
        v[j].i = ids ? ids[j] : (int32_t)j;
    }
    qsort(v, (size_t)n, sizeof(scored_t), cmp_desc);
    int32_t cnt = (int32_t)(n < K ? n : K);
    for (int32_t k = 0; k < cnt; ++k) out_idx[k] = v[k].i;
    qsort(out_idx, (size_t)cnt, sizeof(int32_t), cmp_i32);
    for (int32_t k = cnt; k < K; ++k) out_idx[k] = -1;
    free(v);
    return cnt;
}

/* ------------------------------------------------------------------------ */
/* A8/A9: attention of one query row.                                       */
/* [B §CSA2：三层压缩一次吃满]: entries carry an MLA-style latent shared by  */
/* all heads, so K = V = the dequantised 512-d latent.  The selected main   */
/* entries and the layer's own 8-bit window ([B §CSA2], [A §有界重放的滑动  */
/* 窗口]) form one softmax.  fp64 throughout.                                */
/*   q: [H][D] bf16 bits; kv rows: codes at kv + j*row_stride, scales at    */
/*   kv_scales + j*row_stride; idx: [K] entry ids (-1 = empty);             */
/*   swa: [swa_n][D] E4M3 codes with per-token fp32 scales.                 */
/*   out: [H][D] fp64; lse: [H] (natural log), -inf when no key is seen.   */
/* ------------------------------------------------------------------------ */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

void oracle_attention(const uint16_t *q, int H, int D,
                      const uint8_t *kv_codes, const uint8_t *kv_scales, int64_t kv_row_stride,
                      const int32_t *idx, int32_t K,
                      const uint8_t *swa_codes, const float *swa_scale, int32_t swa_n,
                      double softmax_scale, double *out, double *lse)
{
    int32_t nsel = 0;
    for (int32_t k = 0; k < K; ++k) nsel += idx[k] >= 0;
    int32_t nk = nsel + swa_n;
    double *V = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * D);
    int32_t r = 0;
    for (int32_t k = 0; k < K; ++k) {
        if (idx[k] < 0) continue;
        const uint8_t *c = kv_codes + (int64_t)idx[k] * kv_row_stride;
        const uint8_t *s = kv_scales + (int64_t)idx[k] * kv_row_stride;
        for (int d = 0; d < D; ++d) V[(size_t)r * D + d] = fp4_value(c, s, d);
        ++r;
    }
    for (int32_t t = 0; t < swa_n; ++t, ++r)
        for (int d = 0; d < D; ++d)
            V[(size_t)r * D + d] = oracle_e4m3_value(swa_codes[(size_t)t * D + d]) * (double)swa_scale[t];

    #pragma omp parallel for schedule(static)
    for (int h = 0; h < H; ++h) {
        double *o = out + (size_t)h * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (nk == 0) { lse[h] = -INFINITY; continue; }
        double *z = (double *)malloc(sizeof(double) * nk);
        double m = -INFINITY;
        for (int32_t x = 0; x < nk; ++x) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += bf16_value(q[(size_t)h * D + d]) * V[(size_t)x * D + d];
            z[x] = softmax_scale * acc;
            if (z[x] > m) m = z[x];
        }
        double l = 0.0;
        for (int32_t x = 0; x < nk; ++x) {
            double e = exp(z[x] - m);
            l += e;
            for (int d = 0; d < D; ++d) o[d] += e * V[(size_t)x * D + d];
        }
        for (int d = 0; d < D; ++d) o[d] /= l;
        lse[h] = m + log(l);
        free(z);
    }
    free(V);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
