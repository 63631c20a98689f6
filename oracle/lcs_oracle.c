/*
 * lcs_oracle.c -- plain, slow CPU oracle for the CSA / HCA compressed-attention
 * hot path (DeepSeek-V4 "混合压缩注意力").
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark load it (through oracle/oracle.py).  It shares no code, header,
 * table or constant generator with the CUDA path.
 *
 * Sources (all prose; the pages print no equations):
 *   [p3-2]  "DeepSeek V4 深度解析", section 2 (CSA steps 1-3, HCA paragraph,
 *           mixed-precision KV sentence at the end of the section).
 *   [p3-4]  same page, section 4, "FP4量化感知訓練" paragraph.
 *   [p5-1]  "V3 vs V4" page, inline heading "V4 改进一CSA 与 HCA".
 *   [p5-fp4] same page, inline heading "FP4 为什么能无损".
 *   [p1-g]  podcast show-notes glossary, entries CSA and HCA.
 *
 * Precision: everything that the pages leave open is computed in double and
 * rounded once at the end.  Where a step fixes an fp32 order (the index score
 * chains, the FP4 per-block sums) the oracle follows that order with C's fmaf,
 * which is correctly rounded.  Build with -ffp-contract=off and no fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Number formats.                                                           */
/* A binary format with p significant bits (implicit bit included), minimum  */
/* normal exponent emin (subnormals share the ulp 2^(emin-p+1)) and largest   */
/* finite magnitude maxv.  Rounding is to nearest, ties to even (rint in the  */
/* default rounding mode); saturating formats clamp to +-maxv.               */
/* ------------------------------------------------------------------------ */
static double round_format(double x, int p, int emin, double maxv, int saturate)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);              /* |x| = f * 2^e, 0.5 <= f < 1 */
    int lead = e - 1;          /* exponent of the leading bit */
    if (lead < emin) lead = emin;
    double ulp = ldexp(1.0, lead - (p - 1));
    double r = rint(x / ulp) * ulp;   /* x/ulp is exact: ulp is a power of two */
    if (saturate) {
        if (r > maxv) r = maxv;
        if (r < -maxv) r = -maxv;
    }
    return r;
}

/* bf16: 8 significant bits, emin -126.  Rounding from double directly is a
 * single rounding of the exact value. */
ORC_API double orc_round_bf16(double x) { return round_format(x, 8, -126, 3.3895313892515355e38, 0); }
ORC_API double orc_round_f32(double x) { return (double)(float)x; }

ORC_API uint16_t orc_bf16_bits(double x)
{
    /* x must already be a bf16 value: its float bits end in 16 zero bits. */
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

ORC_API double orc_bf16_value(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* FP8 E4M3 ("fn" variant of the OCP 8-bit float spec): bias 7, 3 mantissa
 * bits, no infinities, 0x7F/0xFF are NaN, largest finite 448. */
ORC_API double orc_round_e4m3(double x) { return round_format(x, 4, -6, 448.0, 1); }

ORC_API double orc_e4m3_value(uint8_t c)
{
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9)            /* subnormal: m/8 * 2^-6 */
                        : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

ORC_API uint8_t orc_e4m3_code(double v)
{
    /* v must be an E4M3 value (output of orc_round_e4m3). */
    uint8_t s = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -6) return s | (uint8_t)(a / ldexp(1.0, -9));   /* subnormal */
    int m = (int)((a / ldexp(1.0, lead) - 1.0) * 8.0);
    return s | (uint8_t)(((lead + 7) << 3) | m);
}

/* FP4 E2M1: bias 1, 1 mantissa bit, values 0, .5, 1, 1.5, 2, 3, 4, 6. */
ORC_API double orc_round_e2m1(double x) { return round_format(x, 2, 0, 6.0, 1); }

ORC_API double orc_e2m1_value(uint8_t nib)
{
    int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

ORC_API uint8_t orc_e2m1_code(double v)
{
    uint8_t s = (v < 0 || (v == 0 && signbit(v))) ? 8 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    if (a == 0.5) return s | 1;
    int e;
    frexp(a, &e);
    int lead = e - 1;                       /* 0, 1 or 2 */
    int m = (int)((a / ldexp(1.0, lead) - 1.0) * 2.0);
    return s | (uint8_t)(((lead + 1) << 1) | m);
}

/* ------------------------------------------------------------------------ */
/* Storage quantisers (the cache-writer side of [p3-2] last paragraph and    */
/* [p3-4]).  The pages fix the formats, not the scale rule; the rules below  */
/* are the adopted reading.                                                  */
/* ------------------------------------------------------------------------ */

/* Mixed-precision KV row: dims [0, d_c) in E4M3 with one fp32 scale per
 * 128-dim block, dims [d_c, d_c + d_r) in bf16.  Row bytes:
 *   d_c codes | 2*d_r bytes bf16 | 4*(d_c/128) bytes fp32 scales.
 * scale = the smallest power of two >= amax/448 (amax/448 in fp32; 1 if amax == 0),
 * code = E4M3(x/scale).  With a power-of-two scale every stored value code*scale
 * is exactly representable in bf16, so widening to bf16 loses nothing. */
ORC_API void orc_quant_kv_fp8(const float* x, int64_t n, int d_c, int d_r, uint8_t* out)
{
    int nb = d_c / 128;
    int64_t row_bytes = d_c + 2 * d_r + 4 * nb;
    for (int64_t i = 0; i < n; ++i) {
        const float* xr = x + i * (d_c + d_r);
        uint8_t* o = out + i * row_bytes;
        for (int b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int j = 0; j < 128; ++j) {
                float a = fabsf(xr[b * 128 + j]);
                if (a > amax) amax = a;
            }
            float t = amax / 448.0f;
            float sc = 1.0f;
            if (t > 0.0f) {
                int e;
                float f = frexpf(t, &e);            /* t = f * 2^e, 0.5 <= f < 1 */
                sc = (f == 0.5f) ? t : ldexpf(1.0f, e);
                if (sc < 0x1p-126f) sc = 0x1p-126f;   /* at least the smallest normal */
            }
            for (int j = 0; j < 128; ++j) {
                float t = xr[b * 128 + j] / sc;
                o[b * 128 + j] = orc_e4m3_code(orc_round_e4m3((double)t));
            }
            memcpy(o + d_c + 2 * d_r + 4 * b, &sc, 4);
        }
        for (int j = 0; j < d_r; ++j) {
            uint16_t h = orc_bf16_bits(orc_round_bf16((double)xr[d_c + j]));
            memcpy(o + d_c + 2 * j, &h, 2);
        }
    }
}

ORC_API void orc_dequant_kv_fp8(const uint8_t* rows, int64_t n, int d_c, int d_r, double* out)
{
    int nb = d_c / 128;
    int64_t row_bytes = d_c + 2 * d_r + 4 * nb;
    for (int64_t i = 0; i < n; ++i) {
        const uint8_t* r = rows + i * row_bytes;
        double* o = out + i * (d_c + d_r);
        for (int b = 0; b < nb; ++b) {
            float sc;
            memcpy(&sc, r + d_c + 2 * d_r + 4 * b, 4);
            for (int j = 0; j < 128; ++j) o[b * 128 + j] = orc_e4m3_value(r[b * 128 + j]) * (double)sc;
        }
        for (int j = 0; j < d_r; ++j) {
            uint16_t h;
            memcpy(&h, r + d_c + 2 * j, 2);
            o[d_c + j] = orc_bf16_value(h);
        }
    }
}

/* FP4 E2M1 with one E4M3 scale per 32 elements ([p3-4]: the indexer's QK path
 * is FP4).  scale = E4M3(amax/6), amax/6 in fp32, 1 if that rounds to 0;
 * code = E2M1(x/scale), x/scale in fp32, saturating at +-6.
 * Layout of n vectors of length d: packed plane n*(d/2) bytes, element 2j in
 * the low nibble of byte j; then the scale plane n*(d/32) bytes. */
ORC_API void orc_quant_fp4(const float* x, int64_t n, int d, uint8_t* packed, uint8_t* scales)
{
    int nb = d / 32;
    for (int64_t i = 0; i < n; ++i) {
        const float* xr = x + i * d;
        for (int b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float a = fabsf(xr[b * 32 + j]);
                if (a > amax) amax = a;
            }
            double scd = orc_round_e4m3((double)(amax / 6.0f));
            if (scd == 0.0) scd = 1.0;
            float sc = (float)scd;
            scales[i * nb + b] = orc_e4m3_code(scd);
            for (int j = 0; j < 32; j += 2) {
                uint8_t lo = orc_e2m1_code(orc_round_e2m1((double)(xr[b * 32 + j] / sc)));
                uint8_t hi = orc_e2m1_code(orc_round_e2m1((double)(xr[b * 32 + j + 1] / sc)));
                packed[i * (d / 2) + (b * 32 + j) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* RoPE (rotate-half / NeoX pairing) on the last d_rope dims of each row.    */
/* Pair (c + i, c + i + d_rope/2), i < d_rope/2, c = d - d_rope, frequency   */
/* theta^(-2i/d_rope), angle = pos * frequency.  The pages name RoPE only    */
/* as the dims kept in bf16 ([p3-2] end); the pairing is the adopted reading. */
/* ------------------------------------------------------------------------ */
ORC_API void orc_rope(double* rows, const int64_t* pos, int64_t n, int d, int d_rope, double theta)
{
    int half = d_rope / 2, c = d - d_rope;
    for (int64_t r = 0; r < n; ++r) {
        double* x = rows + r * d;
        for (int i = 0; i < half; ++i) {
            double freq = pow(theta, -2.0 * i / (double)d_rope);
            double a = (double)pos[r] * freq;
            double cs = cos(a), sn = sin(a);
            double x1 = x[c + i], x2 = x[c + i + half];
            x[c + i] = x1 * cs - x2 * sn;
            x[c + i + half] = x2 * cs + x1 * sn;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Token compressor ([p3-2] CSA step 1; [p5-1] "每 m 个相邻 token 的 KV 用一组 */
/* 带位置偏置的 softmax 权重压成 1 条"; HCA is the same form with m'=128).     */
/* Entry j pools the window of m + overlap tokens t = m*j - overlap + i,     */
/* i = 0 .. m+overlap-1, with weights softmax_i(z_t + bias_i).  Tokens with  */
/* t < 0 come from the tail (the overlap tokens before the chunk) when one   */
/* is given, else they are left out and the softmax runs over the rest.     */
/* RoPE is then applied to the pooled entry at position pos0 + m*j + m - 1.  */
/* One request; x [T, d], x_tail [overlap, d], z [T], z_tail [overlap].      */
/* pool_w (optional) receives the weights, 0 for left-out positions.         */
/* ------------------------------------------------------------------------ */
ORC_API int orc_compress(const double* x, const double* x_tail, const double* z, const double* z_tail,
                         const double* bias, int64_t T, int d, int m, int overlap,
                         int d_rope, double theta, int64_t pos0, double* out, double* pool_w)
{
    if (m <= 0 || overlap < 0 || T % m) return -1;
    int wp = m + overlap;
    int64_t n_out = T / m;
    double* lg = (double*)malloc(sizeof(double) * wp);
    int* ok = (int*)malloc(sizeof(int) * wp);
    for (int64_t j = 0; j < n_out; ++j) {
        double mx = -INFINITY;
        for (int i = 0; i < wp; ++i) {
            int64_t t = m * j - overlap + i;
            ok[i] = (t >= 0) || (x_tail != NULL);
            if (!ok[i]) continue;
            double zt = (t >= 0) ? z[t] : z_tail[overlap + t];
            lg[i] = zt + bias[i];
            if (lg[i] > mx) mx = lg[i];
        }
        double s = 0.0;
        for (int i = 0; i < wp; ++i) {
            if (!ok[i]) continue;
            lg[i] = exp(lg[i] - mx);
            s += lg[i];
        }
        double* e = out + j * d;
        for (int c = 0; c < d; ++c) e[c] = 0.0;
        for (int i = 0; i < wp; ++i) {
            double p = ok[i] ? lg[i] / s : 0.0;
            if (pool_w) pool_w[j * wp + i] = p;
            if (!ok[i]) continue;
            int64_t t = m * j - overlap + i;
            const double* xr = (t >= 0) ? x + t * d : x_tail + (overlap + t) * d;
            for (int c = 0; c < d; ++c) e[c] += p * xr[c];
        }
        if (d_rope > 0) {
            int64_t pos = pos0 + m * j + m - 1;
            orc_rope(e, &pos, 1, d, d_rope, theta);
        }
    }
    free(lg);
    free(ok);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Lightning indexer ([p3-2] CSA step 2: a light, low-rank scorer of every    */
/* compressed entry against the query; [p5-1] same).  Adopted form:          */
/*   score(s) = sum_h w_h * ReLU(qI_h . kI_s)                                */
/* with H_I index heads sharing one index key per entry.                     */
/* ------------------------------------------------------------------------ */

/* fp32 inputs: dot_h = fmaf chain over d from 0; score = fmaf chain over h. */
ORC_API void orc_index_scores_f32(const float* qI, const float* w, const float* kI, int64_t N,
                                  int H, int dI, float* score)
{
    for (int64_t s = 0; s < N; ++s) {
        float acc = 0.0f;
        for (int h = 0; h < H; ++h) {
            float dot = 0.0f;
            for (int c = 0; c < dI; ++c) dot = fmaf(qI[h * dI + c], kI[s * dI + c], dot);
            float r = dot > 0.0f ? dot : 0.0f;
            acc = fmaf(w[h], r, acc);
        }
        score[s] = acc;
    }
}

/* Exact sum of n products a_i*b_i of bf16 values, rounded once to fp32.
 * Products of two bf16 values are exact in double.  If every partial sum is
 * a multiple of 2^L and below 2^(L+53) the double sum is exact; otherwise a
 * base-2^32 big integer holds the exact sum. */
static float exact_dot_to_f32(const double* a, const double* b, int n)
{
    int have = 0, lo = 0, hi = 0;
    for (int i = 0; i < n; ++i) {
        if (a[i] == 0.0 || b[i] == 0.0) continue;
        int ea, eb;
        frexp(a[i], &ea);
        frexp(b[i], &eb);
        /* |a| < 2^ea with 8 significant bits: LSB weight 2^(ea-8). */
        int l = (ea - 8) + (eb - 8), h = ea + eb;
        if (!have) { lo = l; hi = h; have = 1; }
        if (l < lo) lo = l;
        if (h > hi) hi = h;
    }
    if (!have) return 0.0f;
    int nbits = 0;
    while ((1 << nbits) < n) ++nbits;
    if (hi + nbits - lo <= 52) {
        double s = 0.0;
        for (int i = 0; i < n; ++i) s += a[i] * b[i];
        return (float)s;
    }
    /* Big-integer path: value = sum_k limb[k] * 2^(lo + 32k). */
    int nl = (hi + nbits + 2 - lo) / 32 + 2;
    int64_t* limb = (int64_t*)calloc((size_t)nl, sizeof(int64_t));
    for (int i = 0; i < n; ++i) {
        if (a[i] == 0.0 || b[i] == 0.0) continue;
        int ea, eb;
        double fa = frexp(a[i], &ea), fb = frexp(b[i], &eb);
        double sa = ldexp(fa, 8), sb = ldexp(fb, 8);
        if (sa != rint(sa) || sb != rint(sb)) { free(limb); return NAN; }  /* not bf16 values */
        int64_t ma = (int64_t)sa, mb = (int64_t)sb;                       /* exact, |m| < 256 */
        int64_t prod = ma * mb;                                          /* |prod| < 2^16 */
        int sh = (ea - 8) + (eb - 8) - lo;
        int k = sh / 32, r = sh % 32;
        int64_t v = prod * ((int64_t)1 << r);   /* |v| < 2^48 */
        limb[k] += v % ((int64_t)1 << 32);
        limb[k + 1] += v / ((int64_t)1 << 32);
    }
    /* Normalise to digits in [0, 2^32) with a signed top. */
    for (int k = 0; k < nl - 1; ++k) {
        int64_t c = limb[k] >> 32;   /* floor division */
        limb[k] -= c * ((int64_t)1 << 32);
        limb[k + 1] += c;
    }
    int neg = limb[nl - 1] < 0;
    if (neg) {   /* negate the two's-complement number */
        int64_t carry = 1;
        for (int k = 0; k < nl; ++k) {
            int64_t v = ((~limb[k]) & 0xFFFFFFFFLL) + carry;
            carry = v >> 32;
            limb[k] = v & 0xFFFFFFFFLL;
        }
    }
    int top = -1;
    for (int k = nl - 1; k >= 0 && top < 0; --k)
        if (limb[k]) for (int bit = 31; bit >= 0; --bit)
            if ((limb[k] >> bit) & 1) { top = 32 * k + bit; break; }
    float res = 0.0f;
    if (top >= 0) {
        /* Keep 24 significant bits, or fewer if the result is an fp32 subnormal. */
        int cut = top - 23;                      /* bit index of the kept LSB */
        if (lo + cut < -149) cut = -149 - lo;
        if (cut <= 0) {
            double v = 0.0;
            for (int k = nl - 1; k >= 0; --k) v = v * 4294967296.0 + (double)limb[k];
            res = (float)ldexp(v, lo);
        } else {
            #define BIT(i) ((int)((limb[(i) / 32] >> ((i) % 32)) & 1))
            uint64_t mant = 0;
            for (int i = top; i >= cut; --i) mant = (mant << 1) | (uint64_t)BIT(i);
            int rbit = BIT(cut - 1), sticky = 0;
            for (int i = cut - 2; i >= 0 && !sticky; --i) sticky = BIT(i);
            #undef BIT
            if (rbit && (sticky || (mant & 1))) mant += 1;
            res = (float)ldexp((double)mant, lo + cut);
        }
    }
    free(limb);
    return neg ? -res : res;
}

ORC_API float orc_exact_dot_f32(const double* a, const double* b, int n) { return exact_dot_to_f32(a, b, n); }

/* bf16 inputs (given as exact doubles): dot_h = exact dot rounded once to
 * fp32; score = fmaf chain over h, as for fp32. */
ORC_API void orc_index_scores_bf16(const double* qI, const float* w, const double* kI, int64_t N,
                                   int H, int dI, float* score)
{
    for (int64_t s = 0; s < N; ++s) {
        float acc = 0.0f;
        for (int h = 0; h < H; ++h) {
            float dot = exact_dot_to_f32(qI + (int64_t)h * dI, kI + s * dI, dI);
            float r = dot > 0.0f ? dot : 0.0f;
            acc = fmaf(w[h], r, acc);
        }
        score[s] = acc;
    }
}

/* FP4 QK path ([p3-4]; [p5-fp4]).  Both sides are E2M1 with an E4M3 scale per
 * 32-block.  D_b = sum over the block of qcode*kcode is exact (a multiple of
 * 0.25, |D_b| <= 1152).  dot_h = fixed-order fmaf over b of D_b * c_b with
 * c_b = sq_{h,b} * sk_{s,b} (exact: 4-bit by 4-bit significands).  score =
 * fmaf chain over h, then rounded to bf16 ([p5-fp4]: index scores in BF16).
 * q_packed/q_scales: the query quantised by orc_quant_fp4 ([H, dI]). */
ORC_API void orc_index_scores_fp4(const uint8_t* q_packed, const uint8_t* q_scales, const float* w,
                                  const uint8_t* k_packed, const uint8_t* k_scales, int64_t N,
                                  int H, int dI, int round_bf16, double* score)
{
    int nb = dI / 32;
    for (int64_t s = 0; s < N; ++s) {
        float acc = 0.0f;
        for (int h = 0; h < H; ++h) {
            float dot = 0.0f;
            for (int b = 0; b < nb; ++b) {
                double Db = 0.0;
                for (int j = 0; j < 32; ++j) {
                    int e = b * 32 + j;
                    uint8_t qb = q_packed[(int64_t)h * (dI / 2) + e / 2];
                    uint8_t kb = k_packed[s * (dI / 2) + e / 2];
                    uint8_t qn = (e & 1) ? (qb >> 4) : (qb & 15);
                    uint8_t kn = (e & 1) ? (kb >> 4) : (kb & 15);
                    Db += orc_e2m1_value(qn) * orc_e2m1_value(kn);
                }
                float c = (float)(orc_e4m3_value(q_scales[h * nb + b]) * orc_e4m3_value(k_scales[s * nb + b]));
                if (b == 0) dot = (float)Db * c;
                else dot = fmaf((float)Db, c, dot);
            }
            float r = dot > 0.0f ? dot : 0.0f;
            acc = fmaf(w[h], r, acc);
        }
        /* the pages' BF16 index score; the fp32 sum itself when round_bf16 == 0 */
        score[s] = round_bf16 ? orc_round_bf16((double)acc) : (double)acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Top-k ([p3-2] CSA step 2: each query keeps the top-k compressed entries). */
/* The k largest of score[0..n) by (score descending, index ascending), then */
/* returned in ascending index order, padded with -1 up to k.  -0 == +0.     */
/* ------------------------------------------------------------------------ */
/* One per thread: callers may run the oracle on several threads at once. */
static _Thread_local const float* g_sort_scores;
static int cmp_desc(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    float sa = g_sort_scores[a], sb = g_sort_scores[b];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (a < b) ? -1 : (a > b);
}
static int cmp_int(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a < b) ? -1 : (a > b);
}

ORC_API void orc_topk(const float* score, int64_t n, int k, int32_t* idx)
{
    int32_t* ord = (int32_t*)malloc(sizeof(int32_t) * (n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) ord[i] = (int32_t)i;
    g_sort_scores = score;
    qsort(ord, (size_t)n, sizeof(int32_t), cmp_desc);
    int64_t take = n < k ? n : k;
    qsort(ord, (size_t)take, sizeof(int32_t), cmp_int);
    for (int64_t i = 0; i < k; ++i) idx[i] = i < take ? ord[i] : -1;
    free(ord);
}

/* ------------------------------------------------------------------------ */
/* Shared-KV MQA over a row set ([p3-2] "都用共享KV的多查詢注意力"; [p5-1]).   */
/* All H heads attend to the same rows: s_hr = scale * q_h . K_r over all D  */
/* dims, one softmax over the whole row set, o_h = sum_r p_hr V_r with V_r   */
/* the first dv dims of the row.  lse_h = log sum_r exp(s_hr).               */
/* ------------------------------------------------------------------------ */
ORC_API void orc_mqa_rows(const double* q, const double* rows, int64_t R, int H, int D, int dv,
                          double scale, double* out, double* lse)
{
    double* s = (double*)malloc(sizeof(double) * (R > 0 ? R : 1));
    for (int h = 0; h < H; ++h) {
        const double* qh = q + (int64_t)h * D;
        double mx = -INFINITY;
        for (int64_t r = 0; r < R; ++r) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c) acc += qh[c] * rows[r * D + c];
            s[r] = scale * acc;
            if (s[r] > mx) mx = s[r];
        }
        double sum = 0.0;
        for (int64_t r = 0; r < R; ++r) { s[r] = exp(s[r] - mx); sum += s[r]; }
        double* o = out + (int64_t)h * dv;
        for (int c = 0; c < dv; ++c) o[c] = 0.0;
        for (int64_t r = 0; r < R; ++r) {
            double p = s[r] / sum;
            for (int c = 0; c < dv; ++c) o[c] += p * rows[r * D + c];
        }
        if (lse) lse[h] = (R > 0) ? mx + log(sum) : -INFINITY;
        if (R == 0) for (int c = 0; c < dv; ++c) o[c] = 0.0;
    }
    free(s);
}

/* Row set of one query ([p3-2] CSA step 3: the selected compressed entries
 * together with the most recent W raw tokens):
 *   comp rows idx[0..k) that are not -1, then the window rows.
 * The window of a query at absolute position t is every row r of win whose
 * position win_pos0 + r lies in [t - W + 1, t].  With t < 0 ("decode") every
 * row of win is in the window.  Returns the number of rows written. */
static int64_t gather_window(const double* win, int64_t Tw, int64_t win_pos0, int64_t t, int W,
                             int D, double* dst)
{
    int64_t n = 0;
    for (int64_t r = 0; r < Tw; ++r) {
        int64_t p = win_pos0 + r;
        if (t >= 0 && (p > t || p < t - W + 1)) continue;
        memcpy(dst + n * D, win + r * D, sizeof(double) * D);
        ++n;
    }
    return n;
}

ORC_API int64_t orc_csa_attend(const double* q, const double* comp, int64_t Nc, const int32_t* idx, int k,
                               const double* win, int64_t Tw, int64_t win_pos0, int64_t t, int W,
                               int H, int D, int dv, double scale, double* out, double* lse)
{
    double* rows = (double*)malloc(sizeof(double) * (size_t)(k + Tw + 1) * D);
    int64_t R = 0;
    for (int i = 0; i < k; ++i) {
        if (idx[i] < 0) continue;
        if (idx[i] >= Nc) { free(rows); return -1; }
        memcpy(rows + R * D, comp + (int64_t)idx[i] * D, sizeof(double) * D);
        ++R;
    }
    R += gather_window(win, Tw, win_pos0, t, W, D, rows + R * D);
    orc_mqa_rows(q, rows, R, H, D, dv, scale, out, lse);
    free(rows);
    return R;
}

/* HCA ([p3-2] HCA paragraph; [p1-g] "query无需挑选token"): every available
 * compressed entry plus the window, no selection.  n_avail = Nc when t < 0,
 * else min(Nc, floor((t+1)/m)) (entry j is complete once token m*j+m-1 is). */
ORC_API int64_t orc_hca_attend(const double* q, const double* comp, int64_t Nc, int m,
                               const double* win, int64_t Tw, int64_t win_pos0, int64_t t, int W,
                               int H, int D, int dv, double scale, double* out, double* lse)
{
    int64_t na = Nc;
    if (t >= 0) {
        int64_t a = (t + 1) / m;
        if (a < na) na = a;
    }
    double* rows = (double*)malloc(sizeof(double) * (size_t)(na + Tw + 1) * D);
    memcpy(rows, comp, sizeof(double) * (size_t)na * D);
    int64_t R = na + gather_window(win, Tw, win_pos0, t, W, D, rows + na * D);
    orc_mqa_rows(q, rows, R, H, D, dv, scale, out, lse);
    free(rows);
    return R;
}

/* ------------------------------------------------------------------------ */
/* Grouped output projection ([p3-2] "都分分組輸出投影降低計算量"; [p5-1]      */
/* "输出端分组投影省算力").  The H*dv head outputs are split into G groups of  */
/* consecutive heads; group g is projected by its own Wg[g] to dg dims; the  */
/* concatenation is projected by Wo to hidden dims.                          */
/*   o [H*dv], Wg [G, (H/G)*dv, dg], Wo [G*dg, hidden] -> y [hidden].        */
/* ------------------------------------------------------------------------ */
ORC_API void orc_group_oproj(const double* o, const double* Wg, const double* Wo, int H, int dv,
                             int G, int dg, int hidden, double* y)
{
    int gin = (H / G) * dv;
    double* cat = (double*)malloc(sizeof(double) * G * dg);
    for (int g = 0; g < G; ++g)
        for (int c = 0; c < dg; ++c) {
            double acc = 0.0;
            for (int i = 0; i < gin; ++i) acc += o[g * gin + i] * Wg[((int64_t)g * gin + i) * dg + c];
            cat[g * dg + c] = acc;
        }
    for (int c = 0; c < hidden; ++c) {
        double acc = 0.0;
        for (int i = 0; i < G * dg; ++i) acc += cat[i] * Wo[(int64_t)i * hidden + c];
        y[c] = acc;
    }
    free(cat);
}

/* ------------------------------------------------------------------------ */
/* Array helpers for the Python side (rounding of doubles; code decoding).   */
/* fmt: 0 fp32, 1 bf16, 2 E4M3 (saturating), 3 E2M1 (saturating).            */
/* ------------------------------------------------------------------------ */
/* Projection of a token's hidden state in fp32 ([p3-2] CSA steps 1-2: the  */
/* KV and index-key rows, the pooling logits, the index queries and head    */
/* weights are linear in the token's hidden state).  The pages give no      */
/* order; the order of the fused kernels is adopted: out[t][c] is the fma   */
/* chain over i = 0 .. n-1 of h[t][i] * W[i][c] in fp32, from 0 (fmaf is    */
/* correctly rounded).  h [T, n], W [n, d], out [T, d].                      */
/* ------------------------------------------------------------------------ */
ORC_API void orc_project_f32(const float* h, const float* W, int64_t T, int n, int d, float* out)
{
    for (int64_t t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            float acc = 0.0f;
            for (int i = 0; i < n; ++i) acc = fmaf(h[t * n + i], W[(int64_t)i * d + c], acc);
            out[t * d + c] = acc;
        }
}

/* ------------------------------------------------------------------------ */
ORC_API void orc_round_array(const double* x, int64_t n, int fmt, double* out)
{
    for (int64_t i = 0; i < n; ++i) {
        double v = x[i];
        out[i] = fmt == 0 ? orc_round_f32(v) : fmt == 1 ? orc_round_bf16(v)
               : fmt == 2 ? orc_round_e4m3(v) : orc_round_e2m1(v);
    }
}

ORC_API void orc_decode_array(const uint8_t* codes, int64_t n, int fmt, double* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = fmt == 2 ? orc_e4m3_value(codes[i]) : orc_e2m1_value(codes[i] & 15);
}

ORC_API void orc_encode_array(const double* v, int64_t n, int fmt, uint8_t* codes)
{
    for (int64_t i = 0; i < n; ++i)
        codes[i] = fmt == 2 ? orc_e4m3_code(v[i]) : orc_e2m1_code(v[i]);
}
