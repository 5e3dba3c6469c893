/*
 * CSA2 CPU oracle -- TEST INFRASTRUCTURE ONLY (see csa2_ref.h).
 *
 * Compiled with -ffp-contract=off: every fp32 operation below is one IEEE
 * operation with round-to-nearest-even, exactly as written.  Where a floating
 * point value decides an integer code (the cache write), the computation is
 * fp32 in a fixed order; everything else (scores, softmax, attention) is fp64.
 */
#include "csa2_ref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int ref_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ formats */

/* E2M1 (OCP MX v1.0, FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit.
 * Exponent 0 is subnormal: 0 or 0.5.  Eight magnitudes: 0, .5, 1, 1.5, 2, 3, 4, 6
 * (the FP4 section of "DeepSeek-V4.1-Flash, expliqué pas à pas" notes that the
 * format has only eight magnitudes). */
double ref_e2m1_value(unsigned code) {
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* E4M3 (OCP FP8, "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * exponent 0 subnormal; S.1111.111 is NaN; largest finite 448. */
double ref_e4m3_value(unsigned code) {
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* E8M0 (OCP MX v1.0 scale): 2^(code-127); 0xFF is NaN. */
double ref_e8m0_value(unsigned code) {
    return code == 255u ? NAN : ldexp(1.0, (int)code - 127);
}

/* Nearest E2M1 value to v; ties go to the even code (mantissa bit 0); values
 * beyond 6 saturate to 6; the sign bit is kept (a negative value that rounds
 * to zero is code 0x8). */
unsigned ref_e2m1_encode(float v) {
    unsigned sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    unsigned best = 0;
    double bestd = INFINITY;
    for (unsigned c = 0; c < 8; ++c) {
        double d = fabs(ref_e2m1_value(c) - a);
        if (d < bestd || (d == bestd && (c & 1u) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return sign | best;
}

/* Nearest finite E4M3 value to v; ties to the even code; saturates at 448. */
unsigned ref_e4m3_encode(float v) {
    unsigned sign = signbit(v) ? 0x80u : 0u;
    double a = fabs((double)v);
    unsigned best = 0;
    double bestd = INFINITY;
    for (unsigned c = 0; c <= 0x7Eu; ++c) {
        double d = fabs(ref_e4m3_value(c) - a);
        if (d < bestd || (d == bestd && (c & 1u) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return sign | best;
}

/* SWA window in FP8 ("Le cache KV en FP4": the SWA KV stays in FP8, being more
 * sensitive to quantisation).  The pages give no scale, and the FP8 main entry
 * of V4 they cite takes 512 bytes for 512 channels, so none: one E4M3 code per
 * channel, the nearest finite E4M3 value of the input (ref_e4m3_encode: ties to
 * the even code, saturating at 448, sign kept). */
void ref_window_fp8(const float* x, int n, uint8_t* codes) {
    for (int i = 0; i < n; ++i) codes[i] = (uint8_t)ref_e4m3_encode(x[i]);
}

/* OCP MX v1.0 shared scale for FP4 elements: X = floor(log2(amax)) - emax_elem,
 * emax_elem = 2 (6 = 1.5 * 2^2), clamped to the E8M0 range [-127, 127]. */
int ref_mx_shared_exp(float amax) {
    int e;
    (void)frexp((double)amax, &e); /* amax = f * 2^e, f in [0.5, 1) */
    int x = (e - 1) - 2;
    if (x < -127) x = -127;
    if (x > 127) x = 127;
    return x;
}

/* The fp32 exponential both sides of the cache write use (the pages give no
 * compressor formula; a bit-exact cache needs one agreed exp).  Method: Cody &
 * Waite argument reduction by ln 2 split in a 15-bit head (exact products for
 * |n| <= 256) and a tail, then the degree-7 Taylor polynomial of e^r in Horner
 * form with fused multiply-adds, then scaling by 2^n.  |error| <= 2 ulp for
 * results in the normal range. */
float ref_spec_exp(float x) {
    const float log2e = 1.44269502162933349609375f;
    const float ln2_hi = 0.693145751953125f;
    const float ln2_lo = 1.42860682030941723212e-6f;
    if (x > 89.0f) x = 89.0f;
    if (x < -104.0f) x = -104.0f;
    float n = rintf(x * log2e);
    float r = fmaf(-n, ln2_hi, x);
    r = fmaf(-n, ln2_lo, r);
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;
    int n1 = ni / 2, n2 = ni - n1;
    return (p * ldexpf(1.0f, n1)) * ldexpf(1.0f, n2);
}

/* -------------------------------------------------------------- cache write */

/* Ratio-2 compression of one disjoint token pair (2j, 2j+1) (CSA2 chapter of
 * "DeepSeek-V4.1-Flash, expliqué pas à pas": CSA2 drops the overlap between
 * groups): e = w0*x0 + w1*x1 with (w0, w1) = softmax(g0, g1), one
 * scalar gate logit per token.  fp32: w0 = 1/(1 + exp(g1 - g0)), w1 = 1 - w0,
 * e_c = fma(w1, x1_c, w0*x0_c). */
void ref_compress_pair(const float* x0, float g0, const float* x1, float g1, float* e) {
    float E = ref_spec_exp(g1 - g0);
    float w0 = 1.0f / (1.0f + E);
    float w1 = 1.0f - w0;
    for (int c = 0; c < 512; ++c) e[c] = fmaf(w1, x1[c], w0 * x0[c]);
}

/* Main-cache pack ("Le cache KV en FP4": E2M1 values, one E4M3 scale per block
 * of 16 channels, no second global scale -- NVFP4 without its tensor scale).
 * Per block: s = E4M3(amax / 6) rounded to nearest even; code_c = E2M1(e_c / s)
 * (fp32 division, nearest even, saturating at 6); s == 0 gives all-zero codes.
 * Byte layout: channel 2i in the low nibble of byte i, 2i+1 in the high nibble;
 * scale byte j covers channels 16j..16j+15. */
void ref_pack_main(const float* e, uint8_t* codes, uint8_t* scales) {
    memset(codes, 0, 256);
    for (int j = 0; j < 32; ++j) {
        float amax = 0.0f;
        for (int c = 0; c < 16; ++c) {
            float a = fabsf(e[16 * j + c]);
            if (a > amax) amax = a;
        }
        unsigned sc = ref_e4m3_encode(amax / 6.0f);
        scales[j] = (uint8_t)sc;
        float s = (float)ref_e4m3_value(sc);
        for (int c = 0; c < 16; ++c) {
            int ch = 16 * j + c;
            unsigned q = (s == 0.0f) ? 0u : ref_e2m1_encode(e[ch] / s);
            codes[ch >> 1] |= (uint8_t)(q << (4 * (ch & 1)));
        }
    }
}

/* Dequantised main entry (the FP4 entries are decompressed before attention:
 * CSA2 chapter of "DeepSeek-V4.1-Flash, expliqué pas à pas"): E2M1 value times
 * its E4M3 scale; exact in fp32. */
void ref_dequant_main(const uint8_t* codes, const uint8_t* scales, float* out) {
    for (int c = 0; c < 512; ++c) {
        unsigned q = (codes[c >> 1] >> (4 * (c & 1))) & 15u;
        out[c] = (float)(ref_e2m1_value(q) * ref_e4m3_value(scales[c >> 4]));
    }
}

/* OCP MXFP4: blocks of 32 E2M1 elements sharing one E8M0 scale 2^X.
 * amax == 0 gives scale code 0 and all-zero codes; otherwise X per
 * ref_mx_shared_exp and code = E2M1(v * 2^-X) (saturating at 6). */
void ref_mxfp4_quant(const float* v, int n, uint8_t* codes, uint8_t* scales) {
    memset(codes, 0, (size_t)n / 2);
    for (int j = 0; j < n / 32; ++j) {
        float amax = 0.0f;
        for (int c = 0; c < 32; ++c) {
            float a = fabsf(v[32 * j + c]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            scales[j] = 0;
            continue;
        }
        int X = ref_mx_shared_exp(amax);
        scales[j] = (uint8_t)(X + 127);
        float inv = ldexpf(1.0f, -X);
        for (int c = 0; c < 32; ++c) {
            int ch = 32 * j + c;
            unsigned q = ref_e2m1_encode(v[ch] * inv);
            codes[ch >> 1] |= (uint8_t)(q << (4 * (ch & 1)));
        }
    }
}

/* Indexer key = plain projection of the (stored, dequantised) main entry
 * (CSA2 chapter of "DeepSeek-V4.1-Flash, expliqué pas à pas": the indexer key
 * is a simple projection of the main KV), then
 * MXFP4.  k_o = sum_c W[c][o] * deq_c accumulated as fp32 fused multiply-adds
 * in the order c = 0, 1, ..., 511 starting from +0. */
void ref_index_key(const uint8_t* codes, const uint8_t* scales, const float* W, uint8_t* kc,
                   uint8_t* ks) {
    float deq[512], k[128];
    ref_dequant_main(codes, scales, deq);
    for (int o = 0; o < 128; ++o) {
        float acc = 0.0f;
        for (int c = 0; c < 512; ++c) acc = fmaf(W[c * 128 + o], deq[c], acc);
        k[o] = acc;
    }
    ref_mxfp4_quant(k, 128, kc, ks);
}

/* Append T tokens of one sequence to its cache.  Ratio 2: tokens are taken in
 * disjoint pairs in arrival order; an unpaired token waits in the pending slot
 * (it is visible only through the sliding window).  Ratio 1 ("m = 1, sans
 * compression"): each token is an entry.  Returns the new entry count, or -1 if
 * the capacity would be exceeded (nothing is written then). */
int ref_append_tokens(int ratio, const float* x, const float* g, int T, const float* W,
                      int32_t* pend_valid, float* pend_x, float* pend_g, uint8_t* mc, uint8_t* ms,
                      uint8_t* kc, uint8_t* ks, int n_entries, int cap) {
    int have = (ratio == 2) ? *pend_valid : 0;
    int new_entries = (ratio == 2) ? (have + T) / 2 : T;
    if (n_entries + new_entries > cap) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int j = 0; j < new_entries; ++j) {
        float e[512];
        if (ratio == 1) {
            memcpy(e, x + (size_t)j * 512, sizeof(e));
        } else {
            int t0 = 2 * j - have; /* token index of the first element of the pair */
            const float* x0 = (t0 < 0) ? pend_x : x + (size_t)t0 * 512;
            float g0 = (t0 < 0) ? *pend_g : g[t0];
            ref_compress_pair(x0, g0, x + (size_t)(t0 + 1) * 512, g[t0 + 1], e);
        }
        size_t dst = (size_t)(n_entries + j);
        ref_pack_main(e, mc + dst * 256, ms + dst * 32);
        ref_index_key(mc + dst * 256, ms + dst * 32, W, kc + dst * 64, ks + dst * 4);
    }
    if (ratio == 2) {
        int rest = (have + T) % 2;
        if (rest) {
            if (T > 0) {
                memcpy(pend_x, x + (size_t)(T - 1) * 512, 512 * sizeof(float));
                *pend_g = g[T - 1];
            }
            *pend_valid = 1;
        } else {
            *pend_valid = 0;
        }
    }
    return n_entries + new_entries;
}

/* ----------------------------------------------------------------- indexer */

static double mx_elem(const uint8_t* codes, const uint8_t* scales, int c) {
    unsigned q = (codes[c >> 1] >> (4 * (c & 1))) & 15u;
    return ref_e2m1_value(q) * ref_e8m0_value(scales[c >> 5]);
}

/* Indexer score of every entry (the light indexer of the CSA2 chapter scores
 * every main-KV entry from an indexer query and an indexer key):
 * score_e = sum_h w_h * max(0, qhat_h . khat_e), query and key both MXFP4 (the
 * pages: V4 stored the indexer queries and keys in FP4).  fp64; every product
 * of two MXFP4 values is exact. */
void ref_index_scores(const uint8_t* kc, const uint8_t* ks, int N, const uint8_t* qc,
                      const uint8_t* qs, const float* w, int H, double* out) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)H * 128);
    for (int h = 0; h < H; ++h)
        for (int c = 0; c < 128; ++c) qd[h * 128 + c] = mx_elem(qc + h * 64, qs + h * 4, c);
#pragma omp parallel for schedule(static)
    for (int e = 0; e < N; ++e) {
        double kd[128];
        for (int c = 0; c < 128; ++c) kd[c] = mx_elem(kc + (size_t)e * 64, ks + (size_t)e * 4, c);
        double s = 0.0;
        for (int h = 0; h < H; ++h) {
            double dot = 0.0;
            for (int c = 0; c < 128; ++c) dot += qd[h * 128 + c] * kd[c];
            s += (double)w[h] * (dot > 0.0 ? dot : 0.0);
        }
        out[e] = s;
    }
    free(qd);
}

typedef struct {
    double s;
    int32_t i;
} ref_si;

static int cmp_si(const void* a, const void* b) {
    const ref_si* x = (const ref_si*)a;
    const ref_si* y = (const ref_si*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Top-K (the indexer keeps the 512 best entries: "DeepSeek-V4.1-Flash, expliqué
 * pas à pas", attention taxonomy): order all entries by score,
 * higher first, equal scores by lower index first; keep the first min(K, N).
 * Output: the kept indices in increasing index order, then -1 padding to K. */
void ref_topk(const double* scores, int N, int K, int32_t* out) {
    ref_si* v = (ref_si*)malloc(sizeof(ref_si) * (size_t)(N > 0 ? N : 1));
    for (int i = 0; i < N; ++i) {
        v[i].s = scores[i];
        v[i].i = i;
    }
    qsort(v, (size_t)N, sizeof(ref_si), cmp_si);
    int m = N < K ? N : K;
    for (int i = 0; i < m; ++i) out[i] = v[i].i;
    qsort(out, (size_t)m, sizeof(int32_t), cmp_i32);
    for (int i = m; i < K; ++i) out[i] = -1;
    free(v);
}

/* --------------------------------------------------------------- attention */

/* Items one query reads: the selected entries, dequantised (index -1 is
 * skipped), then the valid sliding-window tokens (bf16, exact in fp32).
 * Returns the item count M; items is [M][512] fp32. */
int ref_gather_items(const uint8_t* mc, const uint8_t* ms, int n_entries, const int32_t* idx, int K,
                     const uint16_t* win, int win_len, float* items) {
    int m = 0;
    for (int j = 0; j < K; ++j) {
        int e = idx[j];
        if (e < 0 || e >= n_entries) continue;
        ref_dequant_main(mc + (size_t)e * 256, ms + (size_t)e * 32, items + (size_t)m * 512);
        ++m;
    }
    for (int t = 0; t < win_len; ++t) {
        for (int c = 0; c < 512; ++c) {
            uint32_t u = (uint32_t)win[(size_t)t * 512 + c] << 16;
            float f;
            memcpy(&f, &u, 4);
            items[(size_t)m * 512 + c] = f;
        }
        ++m;
    }
    return m;
}

/* Main attention over the gathered items (CSA2 chapter: the main query reads
 * the selected entries and the layer's local SWA KV): the latent item serves as both key and
 * value (MLA-style shared latent).  Plain softmax in fp64:
 * o_h = sum_j softmax_j(scale * q_h . item_j) * item_j.  M == 0 gives zeros. */
void ref_attention(const float* q, int H, const float* items, int M, double scale, float* out) {
#pragma omp parallel for schedule(static)
    for (int h = 0; h < H; ++h) {
        float* o = out + (size_t)h * 512;
        if (M == 0) {
            for (int c = 0; c < 512; ++c) o[c] = 0.0f;
            continue;
        }
        double* s = (double*)malloc(sizeof(double) * (size_t)M);
        double mx = -INFINITY;
        for (int j = 0; j < M; ++j) {
            double d = 0.0;
            for (int c = 0; c < 512; ++c) d += (double)q[h * 512 + c] * (double)items[(size_t)j * 512 + c];
            s[j] = scale * d;
            if (s[j] > mx) mx = s[j];
        }
        double l = 0.0;
        for (int j = 0; j < M; ++j) {
            s[j] = exp(s[j] - mx);
            l += s[j];
        }
        for (int c = 0; c < 512; ++c) {
            double acc = 0.0;
            for (int j = 0; j < M; ++j) acc += s[j] * (double)items[(size_t)j * 512 + c];
            o[c] = (float)(acc / l);
        }
        free(s);
    }
}
