/*
 * CPU oracle for the K8/V4 quantized-KV decode step.  TEST INFRASTRUCTURE ONLY:
 * only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load
 * this library.  The product path (the CUDA library) never calls it, and the two
 * share no code: no header, no helper, no table.
 *
 * What it follows
 * ---------------
 * The codec is named, not specified, on the pages: the blog.123qwe.co.kr deep
 * dive on magnitudedev/magnitude, section 5 ("core mechanism 3: speculative
 * decoding, quantized KV, prefix sharing"), reports the decode attention unit
 * `attention_decode_k8v4` with keys at 8 bit and values at 4 bit, groups of 32
 * and f16 scales; the trawling.dev "Launch HN: Magnitude" page (section on
 * per-device kernel tuning and performance claims) calls the KV codec
 * TurboQuant-inspired, 8-bit keys / 4-bit values.  The pages give no formula,
 * so the scheme is fixed as follows (each choice is a reading of the pages):
 *
 *   K, per (token, kv-head) vector of D channels:
 *       a = max_c |x_c|                 (fp32, exact)
 *       s = fp16_rn( a / 127.0f )       (IEEE fp32 division, then RNE to fp16)
 *       code_c = clamp( rne( x_c / (float)s ), -127, 127 ),   s == 0 -> code 0
 *   V, per (token, kv-head, group of 32 consecutive channels):
 *       s = fp16_rn( a / 7.0f ),  code_c = clamp( rne( x_c / (float)s ), -8, 7 )
 *       byte j of the group = (code[2j] & 0xF) | ((code[2j+1] & 0xF) << 4)
 *   symmetric: no zero point (the deep dive says "affine"; this library reads
 *   the scheme as symmetric and records the reading).
 *
 *   Attention for query row (query token j of a sequence with n query tokens
 *   and L cached tokens, q-head h, kv-head h / (Hq/Hkv)) over the dequantized
 *   cache k_t = code * s, v_t = code * s, computed in fp64:
 *       z_t = scale * <q, k_t>          for t <= L - n + j  (causal among drafts)
 *       w_t = exp(z_t - max z) / sum exp(z - max z)
 *       out = sum_t w_t v_t,   lse = max z + log(sum exp(z - max z))
 *   The causal rule follows the deep dive's section 5 contract that the
 *   verification of several draft tokens runs as one launch against the cache:
 *   the drafts' K/V are already appended, draft j sees history + drafts 0..j.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 * Every fp32 operation is a single IEEE operation in round-to-nearest-even
 * (x86-64 SSE arithmetic, FLT_EVAL_METHOD == 0).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#if defined(__FLT_EVAL_METHOD__) && __FLT_EVAL_METHOD__ != 0
#error "oracle needs FLT_EVAL_METHOD == 0 (plain single-precision arithmetic)"
#endif

/* ---- fp16 <-> fp32/fp64 ------------------------------------------------
 * The compiler's _Float16 conversion is IEEE binary16 with round-to-nearest-even
 * (gcc on x86-64).  Pinned in tests against numpy's float16 cast.              */
uint16_t mqo_f32_to_f16_bits(float x) {
    _Float16 h = (_Float16)x;
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

double mqo_f16_bits_to_f64(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (double)h;
}

static float f16_bits_to_f32(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (float)h;
}

/* bf16 bits -> fp32: a bf16 value is the top half of an fp32 word (exact). */
float mqo_bf16_bits_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* round half to even in the default rounding mode (FE_TONEAREST) */
static float rne(float x) { return nearbyintf(x); }

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* one symmetric quantization of n values with level count `qmax` (127 or 7) and
 * lower clamp `qmin` (-127 or -8): returns the fp16 scale bits, writes codes.  */
static uint16_t quantize_group(const float* x, int n, float qmax, int qmin, int qmaxi, int* codes) {
    float a = 0.0f;
    for (int c = 0; c < n; c++) {
        float m = fabsf(x[c]);
        if (m > a) a = m;
    }
    float s32 = a / qmax;                     /* IEEE fp32 division          */
    uint16_t sb = mqo_f32_to_f16_bits(s32);   /* RNE to fp16                 */
    float s = f16_bits_to_f32(sb);            /* the stored scale, as fp32   */
    for (int c = 0; c < n; c++) {
        if (s == 0.0f) {
            codes[c] = 0;
        } else {
            float r = rne(x[c] / s);          /* IEEE fp32 division, RNE     */
            if (r != r) r = 0.0f;             /* NaN input: out of domain -> 0 */
            /* r is an integer-valued float; clamp before converting so that
             * huge quotients (subnormal scale) cannot overflow the int cast  */
            if (r > (float)qmaxi) r = (float)qmaxi;
            if (r < (float)qmin) r = (float)qmin;
            codes[c] = clampi((int)r, qmin, qmaxi);
        }
    }
    return sb;
}

/* K: x [n_vec][D] fp32 -> codes [n_vec][D] int8, scales [n_vec] fp16 bits */
void mqo_quantize_k(const float* x, int64_t n_vec, int D, int8_t* codes, uint16_t* scales) {
    int* tmp = (int*)malloc(sizeof(int) * (size_t)D);
    for (int64_t i = 0; i < n_vec; i++) {
        scales[i] = quantize_group(x + i * D, D, 127.0f, -127, 127, tmp);
        for (int c = 0; c < D; c++) codes[i * D + c] = (int8_t)tmp[c];
    }
    free(tmp);
}

/* V: x [n_vec][D] fp32 -> packed [n_vec][D/2] u8, scales [n_vec][D/32] fp16 bits */
void mqo_quantize_v(const float* x, int64_t n_vec, int D, uint8_t* packed, uint16_t* scales) {
    int codes[32];
    const int G = D / 32;
    for (int64_t i = 0; i < n_vec; i++) {
        for (int g = 0; g < G; g++) {
            scales[i * G + g] = quantize_group(x + i * D + g * 32, 32, 7.0f, -8, 7, codes);
            for (int j = 0; j < 16; j++) {
                unsigned lo = (unsigned)codes[2 * j] & 0xFu;
                unsigned hi = (unsigned)codes[2 * j + 1] & 0xFu;
                packed[i * (D / 2) + g * 16 + j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* two's-complement 4-bit field -> int */
static int nibble_to_int(unsigned n) { return (n & 0x8u) ? (int)n - 16 : (int)n; }

/* dequantize: the products are exact in fp64 (8 + 11 and 4 + 11 significant bits) */
void mqo_dequantize_k(const int8_t* codes, const uint16_t* scales, int64_t n_vec, int D, double* out) {
    for (int64_t i = 0; i < n_vec; i++) {
        double s = mqo_f16_bits_to_f64(scales[i]);
        for (int c = 0; c < D; c++) out[i * D + c] = (double)codes[i * D + c] * s;
    }
}

void mqo_dequantize_v(const uint8_t* packed, const uint16_t* scales, int64_t n_vec, int D, double* out) {
    const int G = D / 32;
    for (int64_t i = 0; i < n_vec; i++) {
        for (int c = 0; c < D; c++) {
            uint8_t b = packed[i * (D / 2) + c / 2];
            unsigned nib = (c % 2 == 0) ? (b & 0xFu) : (b >> 4);
            double s = mqo_f16_bits_to_f64(scales[i * G + c / 32]);
            out[i * D + c] = (double)nibble_to_int(nib) * s;
        }
    }
}

/* ---- attention --------------------------------------------------------
 * One sequence.  q [n_q][Hq][D], k, v [L][Hkv][D] (fp64, logical token order),
 * out [n_q][Hq][D], lse [n_q][Hq], weights (nullable) [n_q][Hq][L] (zero for
 * masked positions).  Query j attends to t = 0 .. L - n_q + j.  Rows are
 * independent; they are spread over `n_threads` OpenMP threads (<= 1: serial). */
void mqo_attention_f64(const double* q, const double* k, const double* v, int n_q, int Hq, int Hkv, int D,
                       int64_t L, double scale, double* out, double* lse, double* weights, int n_threads) {
    const int G = Hq / Hkv;
    const int rows = n_q * Hq;
#ifdef _OPENMP
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
    for (int r = 0; r < rows; r++) {
        const int j = r / Hq, h = r % Hq, hk = h / G;
        const int64_t n_vis = L - n_q + j + 1;   /* visible tokens 0 .. n_vis-1 */
        const double* qr = q + (int64_t)r * D;
        double* z = (double*)malloc(sizeof(double) * (size_t)(n_vis > 0 ? n_vis : 1));
        double m = -INFINITY;
        for (int64_t t = 0; t < n_vis; t++) {
            const double* kt = k + (t * Hkv + hk) * (int64_t)D;
            double dot = 0.0;
            for (int c = 0; c < D; c++) dot += qr[c] * kt[c];
            z[t] = scale * dot;
            if (z[t] > m) m = z[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < n_vis; t++) { z[t] = exp(z[t] - m); l += z[t]; }
        double* o = out + (int64_t)r * D;
        for (int c = 0; c < D; c++) o[c] = 0.0;
        for (int64_t t = 0; t < n_vis; t++) {
            const double w = z[t] / l;
            const double* vt = v + (t * Hkv + hk) * (int64_t)D;
            for (int c = 0; c < D; c++) o[c] += w * vt[c];
            if (weights) weights[(int64_t)r * L + t] = w;
        }
        if (weights) for (int64_t t = n_vis; t < L; t++) weights[(int64_t)r * L + t] = 0.0;
        lse[r] = m + log(l);
        free(z);
    }
}

/* Same attention, reading the cache in its quantized form (codes + fp16 scales,
 * logical token order [L][Hkv]) and dequantizing every element on the fly, so
 * that long caches need no fp64 copy.  Identical arithmetic to dequantize +
 * mqo_attention_f64 (k = code * s is exact, the sums run in the same order).   */
void mqo_attention_quant_f64(const double* q, const int8_t* kc, const uint16_t* ks, const uint8_t* vp,
                             const uint16_t* vs, int n_q, int Hq, int Hkv, int D, int64_t L, double scale,
                             double* out, double* lse, int n_threads) {
    const int G = Hq / Hkv;
    const int NG = D / 32;
    const int rows = n_q * Hq;
#ifdef _OPENMP
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
    for (int r = 0; r < rows; r++) {
        const int j = r / Hq, h = r % Hq, hk = h / G;
        const int64_t n_vis = L - n_q + j + 1;
        const double* qr = q + (int64_t)r * D;
        double* z = (double*)malloc(sizeof(double) * (size_t)(n_vis > 0 ? n_vis : 1));
        double* vt = (double*)malloc(sizeof(double) * (size_t)D);
        double m = -INFINITY;
        for (int64_t t = 0; t < n_vis; t++) {
            const int64_t vec = t * Hkv + hk;
            const double s = mqo_f16_bits_to_f64(ks[vec]);
            double dot = 0.0;
            for (int c = 0; c < D; c++) dot += qr[c] * ((double)kc[vec * D + c] * s);
            z[t] = scale * dot;
            if (z[t] > m) m = z[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < n_vis; t++) { z[t] = exp(z[t] - m); l += z[t]; }
        double* o = out + (int64_t)r * D;
        for (int c = 0; c < D; c++) o[c] = 0.0;
        for (int64_t t = 0; t < n_vis; t++) {
            const int64_t vec = t * Hkv + hk;
            for (int c = 0; c < D; c++) {
                uint8_t b = vp[vec * (D / 2) + c / 2];
                unsigned nib = (c % 2 == 0) ? (b & 0xFu) : (b >> 4);
                vt[c] = (double)nibble_to_int(nib) * mqo_f16_bits_to_f64(vs[vec * NG + c / 32]);
            }
            const double w = z[t] / l;
            for (int c = 0; c < D; c++) o[c] += w * vt[c];
        }
        lse[r] = m + log(l);
        free(vt);
        free(z);
    }
}

int mqo_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- history-based drafting (n-gram lookup over the token history) -------------
 * The deep dive (section 5, the drafting guarantees) lists history-based drafters
 * among the drafters whose step costs only the bytes they read; it gives no
 * algorithm.  Reading: propose the tokens that followed the most recent earlier
 * occurrence of the history's last n tokens.
 *   match i: 0 <= i < L - n and tokens[i + j] == tokens[L - n + j] for j < n
 *   i* = the largest match; drafts[j] = tokens[i* + n + j] for j < min(k, L - i* - n)
 * Returns the number of drafts (0 when L <= n or nothing matches).  Written as the
 * definition: candidates from the latest down, the first full match wins.          */
int mqo_draft_ngram(const int32_t* tokens, int32_t L, int32_t n, int32_t k, int32_t* drafts) {
    if (L <= n || n < 1 || k < 1) return 0;
    for (int32_t i = L - n - 1; i >= 0; i--) {
        int same = 1;
        for (int32_t j = 0; j < n && same; j++) same = tokens[i + j] == tokens[L - n + j];
        if (!same) continue;
        int32_t cnt = L - i - n;
        if (cnt > k) cnt = k;
        for (int32_t j = 0; j < cnt; j++) drafts[j] = tokens[i + n + j];
        return cnt;
    }
    return 0;
}
