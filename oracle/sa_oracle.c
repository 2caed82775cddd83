/*
 * sa_oracle.c -- plain, slow, fp64 CPU oracle for CSA + HCA hybrid attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or execute this file: only the tests, the smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA library and includes no CUDA header.
 *
 * Source of the method: "DeepSeek-V4: Towards Highly Efficient Million-Token
 * Context Intelligence Review" (dimensionstp.github.io), section 3-2 (2)
 * "Hybrid attention with CSA and HCA" and its component table: CSA turns
 * every 4 tokens into one compressed entry and keeps a sparse top-k of the
 * entries; HCA turns every 128 tokens into one entry and attends densely; the
 * compressed K/V may be stored in FP8 (the "Mixed KV storage" row).  The page
 * leaves the pooling operator, the indexer formula and all rounding open; the
 * readings implemented here are:
 *   - pooling = arithmetic mean of each aligned, complete block of m tokens,
 *     summed in fp64 in ascending token order, times (1/m), rounded once from
 *     fp64 to bf16 (round to nearest even); an incomplete tail is excluded;
 *   - fp8 = e4m3 codes with one fp32 scale per 64 consecutive entries,
 *     scale = fp32(amax / 448) (1 if amax == 0),
 *     code = e4m3_rne_satfinite(fp32(x / scale));
 *   - index score = fp32( sum_i qI[i] * Ic[j][i] ), the sum taken in fp64 in
 *     ascending i (each bf16 x bf16 product is exact in fp64); -0 -> +0;
 *   - top-k = the k entries with the largest (score, -index), reported in
 *     ascending index order, padded with -1;
 *   - attention = softmax(scale * q.K^T) V per head, in fp64, scale
 *     1/sqrt(128) unless the caller gives another, lse = log sum exp.
 *   - causal visibility: a query at token position t sees compressed entry c
 *     iff (c + 1) * m <= t.
 *
 * All bf16 / e4m3 values travel as raw bit patterns (uint16 / uint8).
 * Build: gcc -O2 -fPIC -shared -ffp-contract=off -o liboracle.so sa_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------- */
/* Number formats, written from their definitions.                          */
/* bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.           */
/* e4m3 (the "fn" variant): 1 sign, 4 exponent bits (bias 7), 3 fraction    */
/* bits, no infinities, S.1111.111 is NaN, largest finite 1.75 * 2^8 = 448. */
/* ---------------------------------------------------------------------- */

double or_bf16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xFF;
    int f = h & 0x7F;
    double v;
    if (e == 0xFF) {
        v = (f == 0) ? INFINITY : NAN;
    } else if (e == 0) {
        v = ldexp((double)f, -126 - 7); /* subnormal */
    } else {
        v = ldexp(1.0 + (double)f / 128.0, e - 127);
    }
    return sign ? -v : v;
}

/* Round a double to the nearest bf16, ties to even, in one step. */
uint16_t or_bf16_from_double(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e2;
    (void)frexp(a, &e2);           /* a = f * 2^e2, f in [0.5, 1) */
    int ex = e2 - 1;               /* floor(log2 a) */
    if (ex < -126) ex = -126;      /* below the normal range the spacing is fixed */
    double quantum = ldexp(1.0, ex - 7);
    double n = nearbyint(a / quantum); /* a / quantum is exact; default mode = ties-to-even */
    double y = n * quantum;
    if (y >= ldexp(1.0, 128)) return sign | 0x7F80; /* rounds past the largest finite */
    if (y < ldexp(1.0, -126)) {
        return sign | (uint16_t)(y / ldexp(1.0, -133)); /* subnormal (or zero) */
    }
    (void)frexp(y, &e2);
    int ey = e2 - 1;
    int frac = (int)((y / ldexp(1.0, ey) - 1.0) * 128.0);
    return sign | (uint16_t)((ey + 127) << 7) | (uint16_t)frac;
}

double or_e4m3_to_double(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int f = c & 0x7;
    double v;
    if (e == 0xF && f == 0x7) {
        v = NAN;
    } else if (e == 0) {
        v = ldexp((double)f, -6 - 3); /* subnormal */
    } else {
        v = ldexp(1.0 + (double)f / 8.0, e - 7);
    }
    return sign ? -v : v;
}

/* Round to the nearest e4m3 value, ties to even, then clamp to +-448. */
uint8_t or_e4m3_from_double_satfinite(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7E;
    int e2;
    (void)frexp(a, &e2);
    int ex = e2 - 1;
    if (ex < -6) ex = -6;
    if (ex > 8) ex = 8;            /* anything this large clamps below anyway */
    double quantum = ldexp(1.0, ex - 3);
    double n = nearbyint(a / quantum);
    double y = n * quantum;
    if (y > 448.0) y = 448.0;
    if (y < ldexp(1.0, -6)) {
        return sign | (uint8_t)(y / ldexp(1.0, -9));
    }
    (void)frexp(y, &e2);
    int ey = e2 - 1;
    int frac = (int)((y / ldexp(1.0, ey) - 1.0) * 8.0);
    return sign | (uint8_t)((ey + 7) << 3) | (uint8_t)frac;
}

/* ---------------------------------------------------------------------- */
/* O1: sequence-dimension compression (mean pooling of aligned blocks).     */
/* x: [L][d] bf16 bits; out: [L/m][d] bf16 bits.  Returns n = floor(L/m).   */
/* ---------------------------------------------------------------------- */
int64_t or_compress(const uint16_t* x, int64_t L, int d, int m, uint16_t* out) {
    int64_t n = L / m;
    double inv_m = 1.0 / (double)m;
    for (int64_t c = 0; c < n; ++c) {
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int64_t t = c * m; t < c * m + m; ++t) s += or_bf16_to_double(x[t * d + i]);
            out[c * d + i] = or_bf16_from_double(s * inv_m);
        }
    }
    return n;
}

/* ---------------------------------------------------------------------- */
/* O2: e4m3 storage with one fp32 scale per 64 consecutive entries.         */
/* xc: [n][d] bf16 bits; codes: [n][d]; scales: [ceil(n/64)].               */
/* ---------------------------------------------------------------------- */
void or_fp8_quantize(const uint16_t* xc, int64_t n, int d, uint8_t* codes, float* scales) {
    for (int64_t g = 0; g * 64 < n; ++g) {
        int64_t lo = g * 64, hi = lo + 64 < n ? lo + 64 : n;
        double amax = 0.0;
        for (int64_t j = lo; j < hi; ++j)
            for (int i = 0; i < d; ++i) {
                double v = fabs(or_bf16_to_double(xc[j * d + i]));
                if (v > amax) amax = v;
            }
        float s = (amax == 0.0) ? 1.0f : (float)(amax / 448.0);
        scales[g] = s;
        for (int64_t j = lo; j < hi; ++j)
            for (int i = 0; i < d; ++i) {
                float q = (float)(or_bf16_to_double(xc[j * d + i]) / (double)s);
                codes[j * d + i] = or_e4m3_from_double_satfinite((double)q);
            }
    }
}

/* ---------------------------------------------------------------------- */
/* O3: CSA indexer scores.  qI: [dI] bf16; Ic: [n][dI] bf16; s: [n] fp32.   */
/* ---------------------------------------------------------------------- */
void or_index_scores(const uint16_t* qI, const uint16_t* Ic, int64_t n, int dI, float* s) {
    double q[1024];
    for (int i = 0; i < dI; ++i) q[i] = or_bf16_to_double(qI[i]);
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dI; ++i) acc += q[i] * or_bf16_to_double(Ic[j * dI + i]);
        float r = (float)acc;
        if (r == 0.0f) r = 0.0f; /* -0 -> +0 */
        s[j] = r;
    }
}

/* ---------------------------------------------------------------------- */
/* O4: top-k by (score descending, index ascending), output ascending.      */
/* ---------------------------------------------------------------------- */
typedef struct { float s; int32_t j; } or_pair;

static int or_cmp_rank(const void* a, const void* b) {
    const or_pair* x = (const or_pair*)a;
    const or_pair* y = (const or_pair*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int or_cmp_int(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x < y) ? -1 : (x > y);
}

/* s: scores of entries 0..n_visible-1.  idx: [k].  Returns the count. */
int32_t or_topk(const float* s, int64_t n_visible, int32_t k, int32_t* idx) {
    int64_t cnt = n_visible < k ? n_visible : k;
    if (cnt > 0) {
        or_pair* p = (or_pair*)malloc(sizeof(or_pair) * (size_t)n_visible);
        for (int64_t j = 0; j < n_visible; ++j) { p[j].s = s[j]; p[j].j = (int32_t)j; }
        qsort(p, (size_t)n_visible, sizeof(or_pair), or_cmp_rank);
        for (int64_t r = 0; r < cnt; ++r) idx[r] = p[r].j;
        free(p);
        qsort(idx, (size_t)cnt, sizeof(int32_t), or_cmp_int);
    }
    for (int64_t r = cnt; r < k; ++r) idx[r] = -1;
    return (int32_t)cnt;
}

/* ---------------------------------------------------------------------- */
/* O5: softmax attention of H query heads over a list of cache rows.        */
/* q: [H][d] bf16.  Rows come from a bf16 cache (kv_fp8 == 0: K, V are      */
/* [N][d] bf16 bits) or an e4m3 cache (kv_fp8 == 1: K, V are [N][d] codes   */
/* and ks, vs are the per-64-entry scales).  rows: [nrows] entry indices.   */
/* out: [H][d] fp64; lse: [H]; p: optional [H][nrows] weights.              */
/* ---------------------------------------------------------------------- */
static double or_kv_value(const void* base, const float* scales, int kv_fp8, int64_t j, int d, int i) {
    if (kv_fp8) {
        const uint8_t* c = (const uint8_t*)base;
        return or_e4m3_to_double(c[j * d + i]) * (double)scales[j / 64];
    }
    const uint16_t* h = (const uint16_t*)base;
    return or_bf16_to_double(h[j * d + i]);
}

void or_attention(const uint16_t* q, int H, int d,
                  const void* K, const float* ks, const void* V, const float* vs, int kv_fp8,
                  const int32_t* rows, int64_t nrows, double scale,
                  double* out, double* lse, double* p) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1));
    for (int h = 0; h < H; ++h) {
        double* o = out + (int64_t)h * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (nrows == 0) {
            lse[h] = -INFINITY;
            continue;
        }
        double zmax = -INFINITY;
        for (int64_t r = 0; r < nrows; ++r) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += or_bf16_to_double(q[(int64_t)h * d + i]) * or_kv_value(K, ks, kv_fp8, rows[r], d, i);
            z[r] = acc * scale;
            if (z[r] > zmax) zmax = z[r];
        }
        double l = 0.0;
        for (int64_t r = 0; r < nrows; ++r) {
            z[r] = exp(z[r] - zmax);
            l += z[r];
        }
        for (int64_t r = 0; r < nrows; ++r) {
            double w = z[r] / l;
            if (p) p[(int64_t)h * nrows + r] = w;
            for (int i = 0; i < d; ++i) o[i] += w * or_kv_value(V, vs, kv_fp8, rows[r], d, i);
        }
        lse[h] = zmax + log(l);
    }
    free(z);
}

/* ---------------------------------------------------------------------- */
/* O6: one sequence, one query, both branches, from already-compressed      */
/* caches.  t = the query's token position (decode: t = L, the cache's raw  */
/* length).  CSA visible set {c : (c+1)*4 <= t}, top-k by the indexer, then */
/* attention over the selected rows; HCA visible set {c : (c+1)*128 <= t}.  */
/* The compression blocks m_csa / m_hca are parameters so that tests can    */
/* reduce the method to dense attention (m = 1).                            */
/* ---------------------------------------------------------------------- */
void or_hybrid_query(const uint16_t* q, const uint16_t* qI, int H, int d, int dI, int64_t t,
                     int m_csa, const void* ck, const float* cks, const void* cv, const float* cvs,
                     const uint16_t* cidx, int64_t n_csa,
                     int m_hca, const void* hk, const float* hks, const void* hv, const float* hvs,
                     int64_t n_hca, int kv_fp8, int32_t topk, double scale,
                     int32_t* idx_out, int32_t* cnt_out,
                     double* out_csa, double* lse_csa, double* out_hca, double* lse_hca) {
    int64_t vis_c = t / m_csa;
    if (vis_c > n_csa) vis_c = n_csa;
    float* s = (float*)malloc(sizeof(float) * (size_t)(vis_c > 0 ? vis_c : 1));
    or_index_scores(qI, cidx, vis_c, dI, s);
    int32_t cnt = or_topk(s, vis_c, topk, idx_out);
    free(s);
    *cnt_out = cnt;
    or_attention(q, H, d, ck, cks, cv, cvs, kv_fp8, idx_out, cnt, scale, out_csa, lse_csa, NULL);

    int64_t vis_h = t / m_hca;
    if (vis_h > n_hca) vis_h = n_hca;
    int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(vis_h > 0 ? vis_h : 1));
    for (int64_t c = 0; c < vis_h; ++c) rows[c] = (int32_t)c;
    or_attention(q, H, d, hk, hks, hv, hvs, kv_fp8, rows, vis_h, scale, out_hca, lse_hca, NULL);
    free(rows);
}

/* ====================================================================== */
/* Low-precision storage on the CSA path ("DeepSeek-V4 ... Review",        */
/* section 3-2 (2), the "Mixed KV storage" row of the component table,     */
/* and section 3-2 (4): FP4 on the CSA indexer QK path).  The pages name   */
/* the formats only; the readings implemented below are:                   */
/*   - indexer FP4 = OCP Microscaling MXFP4: e2m1 elements in blocks of 32 */
/*     consecutive indexer dims, one E8M0 (power of two) scale per block,  */
/*     X = 2^(floor(log2 amax) - 2) with the exponent clamped to           */
/*     [-127, 127] (E8M0 code 0 when amax == 0), element =                 */
/*     e2m1_rne_satfinite(x / X); both the query and the compressed keys   */
/*     are quantized this way;                                             */
/*   - FP4 index score = fp32_rne of the exact real sum over the two       */
/*     blocks of X_q * X_k * sum_i e2m1(q_i) * e2m1(k_i);                   */
/*   - mixed KV storage = the last d_rope dims of each K entry kept in     */
/*     bf16 (the rotary dims), the other K dims and all of V in e4m3 with  */
/*     the per-64-entry scale of O2 taken over the stored-e4m3 dims only.  */
/* ====================================================================== */

/* e2m1: 1 sign bit, 2 exponent bits (bias 1), 1 fraction bit; no inf or   */
/* NaN.  Magnitudes: 0, 0.5 (the subnormal), 1, 1.5, 2, 3, 4, 6.            */
double or_e2m1_to_double(uint8_t c) {
    int sign = (c >> 3) & 1;
    int e = (c >> 1) & 0x3;
    int f = c & 0x1;
    double v = (e == 0) ? 0.5 * (double)f : ldexp(1.0 + 0.5 * (double)f, e - 1);
    return sign ? -v : v;
}

/* Nearest e2m1 value, ties to an even fraction bit, clamped to +-6. */
uint8_t or_e2m1_from_double_satfinite(double x) {
    uint8_t sign = signbit(x) ? 0x8 : 0;
    if (isnan(x)) return sign | 0x7;  /* no NaN in e2m1: saturate */
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7;
    int e2;
    (void)frexp(a, &e2);
    int ex = (a == 0.0) ? 0 : e2 - 1;  /* floor(log2 a) */
    if (ex < 0) ex = 0;                /* spacing 0.5 below 2 (subnormal + first binade) */
    if (ex > 2) ex = 2;
    double quantum = ldexp(1.0, ex - 1);
    double y = nearbyint(a / quantum) * quantum;
    if (y > 6.0) y = 6.0;
    if (y < 1.0) return sign | (uint8_t)(y * 2.0);  /* 0 or the subnormal 0.5 */
    (void)frexp(y, &e2);
    int ey = e2 - 1;                                  /* 0, 1 or 2 */
    int frac = (int)((y / ldexp(1.0, ey) - 1.0) * 2.0);
    return sign | (uint8_t)((ey + 1) << 1) | (uint8_t)frac;
}

/* E8M0: an unsigned biased exponent, value 2^(c - 127); 0xFF is NaN. */
double or_e8m0_to_double(uint8_t c) {
    if (c == 0xFF) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* MXFP4 quantization of rows of bf16 values.  x: [n][d] bf16 bits, d a     */
/* multiple of 32.  codes: [n][d/2], element 2i in the low nibble of byte i */
/* and element 2i+1 in the high nibble; scales: [n][d/32] E8M0 codes.       */
void or_mxfp4_quantize(const uint16_t* x, int64_t n, int d, uint8_t* codes, uint8_t* scales) {
    for (int64_t j = 0; j < n; ++j) {
        for (int b = 0; b < d / 32; ++b) {
            const uint16_t* xb = x + j * d + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double v = fabs(or_bf16_to_double(xb[i]));
                if (v > amax) amax = v;
            }
            int se;
            if (amax == 0.0) {
                se = -127;
            } else {
                int e2;
                (void)frexp(amax, &e2);
                se = (e2 - 1) - 2;  /* floor(log2 amax) - (largest e2m1 exponent) */
                if (se < -127) se = -127;
                if (se > 127) se = 127;
            }
            scales[j * (d / 32) + b] = (uint8_t)(se + 127);
            double X = ldexp(1.0, se);
            for (int i = 0; i < 32; ++i) {
                uint8_t c = or_e2m1_from_double_satfinite(or_bf16_to_double(xb[i]) / X);
                int64_t byte = j * (d / 2) + b * 16 + i / 2;
                if (i % 2 == 0) codes[byte] = c;
                else codes[byte] |= (uint8_t)(c << 4);
            }
        }
    }
}

static double or_mxfp4_elem(const uint8_t* codes, int64_t row, int d, int i) {
    uint8_t byte = codes[row * (d / 2) + i / 2];
    return or_e2m1_to_double((i % 2 == 0) ? (byte & 0xF) : (byte >> 4));
}

/* FP4 index scores.  qc/qs: one MXFP4 query ([d/2] codes, [d/32] scales);  */
/* kc/ks: n MXFP4 key rows.  Each block's dot product is a multiple of 1/4  */
/* below 2^11 in magnitude and is exact in fp64, as is its product with the */
/* two power-of-two scales; the sum of the two block terms is exact in fp64 */
/* whenever their exponents lie within 40 of each other.  Otherwise the     */
/* smaller term is below 2^-27 of the larger, which has at most 13          */
/* significant bits, and rounding the fp64 sum to fp32 gives the larger     */
/* term -- the correctly rounded result -- in the normal fp32 range.        */
void or_mxfp4_index_scores(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                           int64_t n, int d, float* s) {
    for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int b = 0; b < d / 32; ++b) {
            double blk = 0.0;
            for (int i = b * 32; i < b * 32 + 32; ++i)
                blk += or_mxfp4_elem(qc, 0, d, i) * or_mxfp4_elem(kc, j, d, i);
            acc += blk * or_e8m0_to_double(qs[b]) * or_e8m0_to_double(ks[j * (d / 32) + b]);
        }
        float r = (float)acc;
        if (r == 0.0f) r = 0.0f; /* -0 -> +0 */
        s[j] = r;
    }
}

/* Mixed KV storage of one compressed K tensor.  xc: [n][d] bf16 bits.      */
/* codes: [n][d - d_rope] e4m3 for dims [0, d - d_rope); scales:            */
/* [ceil(n/64)] fp32 over those dims (the O2 rule); rope: [n][d_rope] bf16  */
/* bits, dims [d - d_rope, d) unchanged.                                    */
void or_mixed_quantize(const uint16_t* xc, int64_t n, int d, int d_rope,
                       uint8_t* codes, float* scales, uint16_t* rope) {
    int dn = d - d_rope;
    uint16_t* nope = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n > 0 ? n : 1) * (size_t)(dn > 0 ? dn : 1));
    for (int64_t j = 0; j < n; ++j) {
        for (int i = 0; i < dn; ++i) nope[j * dn + i] = xc[j * d + i];
        for (int i = 0; i < d_rope; ++i) rope[j * d_rope + i] = xc[j * d + dn + i];
    }
    if (dn > 0) or_fp8_quantize(nope, n, dn, codes, scales);
    free(nope);
}

/* One stored K or V tensor for or_attention_kv.  mode 0: bf16 [N][d];      */
/* mode 1: e4m3 [N][d] + scales; mode 2: mixed (e4m3 [N][d - d_rope] +      */
/* scales, then bf16 rope [N][d_rope]).                                     */
static double or_kv_elem(int mode, const void* base, const float* scales, const uint16_t* rope, int d_rope,
                         int64_t j, int d, int i) {
    if (mode == 0) return or_bf16_to_double(((const uint16_t*)base)[j * d + i]);
    if (mode == 1) return or_e4m3_to_double(((const uint8_t*)base)[j * d + i]) * (double)scales[j / 64];
    int dn = d - d_rope;
    if (i >= dn) return or_bf16_to_double(rope[j * d_rope + (i - dn)]);
    return or_e4m3_to_double(((const uint8_t*)base)[j * dn + i]) * (double)scales[j / 64];
}

/* O5 with K and V each in any of the storage modes above. */
void or_attention_kv(const uint16_t* q, int H, int d,
                     int k_mode, const void* K, const float* ks, const uint16_t* k_rope,
                     int v_mode, const void* V, const float* vs, const uint16_t* v_rope, int d_rope,
                     const int32_t* rows, int64_t nrows, double scale,
                     double* out, double* lse) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1));
    for (int h = 0; h < H; ++h) {
        double* o = out + (int64_t)h * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (nrows == 0) {
            lse[h] = -INFINITY;
            continue;
        }
        double zmax = -INFINITY;
        for (int64_t r = 0; r < nrows; ++r) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += or_bf16_to_double(q[(int64_t)h * d + i]) *
                       or_kv_elem(k_mode, K, ks, k_rope, d_rope, rows[r], d, i);
            z[r] = acc * scale;
            if (z[r] > zmax) zmax = z[r];
        }
        double l = 0.0;
        for (int64_t r = 0; r < nrows; ++r) {
            z[r] = exp(z[r] - zmax);
            l += z[r];
        }
        for (int64_t r = 0; r < nrows; ++r) {
            double w = z[r] / l;
            for (int i = 0; i < d; ++i) o[i] += w * or_kv_elem(v_mode, V, vs, v_rope, d_rope, rows[r], d, i);
        }
        lse[h] = zmax + log(l);
    }
    free(z);
}
