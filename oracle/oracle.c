/*
 * CPU oracle for the MoE layer forward over quantised experts.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call this code;
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark do.
 * It shares no source, header, table or helper with the CUDA path.
 *
 * It is a plain, slow, obviously correct restatement of what the layer
 * computes, in fp32 (fp64 where noted), with sequential sums and no blocking
 * or fusion. Sources (page titles as printed on the pages):
 *   - "FreeToken: UC Berkeley Brings 753B GLM-5.2 MoE Inference to Consumer
 *     Hardware", section "Reported Numbers and Ecosystem Position": the expert
 *     formats MXFP4, NVFP4, FP8 and BF16.
 *   - winzheng.com "FreeToken ... 753B local inference MoE", section "Why Now
 *     of All Times": a token activates a few routed experts per layer (top-k
 *     routing); the experts are "loaded on demand".
 *   - The same page, section "FreeToken's Three-Layer Mechanism": the global
 *     LRU expert cache (simulated in lru.py, not here).
 * The pages give no formula for the router, the gating, the FFN or the
 * combine. This file takes the plainest standard reading of a top-k softmax
 * SwiGLU MoE layer; every reading is marked READING below.
 *
 * Format definitions (decode only; the encoders live in the input generator):
 *   E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit, exponent 0 subnormal.
 *   E8M0: 8-bit unsigned exponent, value 2^(e-127), 0xFF is NaN.
 *   E4M3 (the "FN" variant): sign, 4 exponent bits (bias 7), 3 mantissa bits,
 *         exponent 0 subnormal, S.1111.111 NaN, no infinity, max 448.
 *   MXFP4 = E2M1 * E8M0 (one scale per 32 elements along K).
 *   NVFP4 = (E2M1 * E4M3) * fp32 tensor scale (one E4M3 per 16 along K).
 *   FP8   = E4M3 * fp32 (one scale per row and 128 elements along K).
 *   READING: two E2M1 codes per byte, the low nibble holds the lower K index.
 *
 * Pins: the pages print no layer-level values to compare against, so every
 * function here is pinned by the tests to something other than itself: hand
 * worked fixtures (E2M1 table, an MXFP4 row), library decoders (torch float8
 * E4M3 / E8M0, bf16 rounding), closed forms (fp64 matmul rounded once, the
 * softmax ratios, a dense SwiGLU MLP at k = E = 1), invariants (a stable
 * counting sort, power-of-two scale steps) and fp64 brute force per token.
 * Planted mistakes in a copy of this file are each caught by one of them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OF_BF16 = 0, OF_FP8 = 1, OF_MXFP4 = 2, OF_NVFP4 = 3 };
enum { ACT_A16 = 0, ACT_A4 = 1 };

/* ---------------------------------------------------------------- scalars */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a binary32 to bf16, to nearest, ties to even (NaN kept quiet). */
static uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

double oracle_bf16_round(double v) { return bf16_to_f32(f32_to_bf16((float)v)); }

/* E2M1 from its definition (see header). */
double oracle_e2m1(int code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E8M0 from its definition. */
double oracle_e8m0(int code) {
    code &= 0xff;
    if (code == 0xff) return NAN;
    return ldexp(1.0, code - 127);
}

/* E4M3 ("FN") from its definition. */
double oracle_e4m3(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp(m / 8.0, -6);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* ------------------------------------------------------------ dequantise */

/* Dequantise one expert tensor [rows, K] of format fmt into fp32.
 * w: bf16 bits / E4M3 codes / packed E2M1 codes, row-major, K contiguous.
 * scale: fp32 [rows][K/128] (FP8), E8M0 [rows][K/32] (MXFP4), E4M3 [rows][K/16] (NVFP4).
 * tscale: NVFP4 per-tensor fp32 scale. Returns 0, or -1 on a bad format/shape. */
int oracle_dequant(int fmt, int rows, int K, const void *w, const void *scale, float tscale, float *out) {
    for (int r = 0; r < rows; ++r) {
        for (int c = 0; c < K; ++c) {
            float v;
            size_t i = (size_t)r * K + c;
            if (fmt == OF_BF16) {
                v = bf16_to_f32(((const uint16_t *)w)[i]);
            } else if (fmt == OF_FP8) {
                if (K % 128) return -1;
                float q = (float)oracle_e4m3(((const uint8_t *)w)[i]);
                float s = ((const float *)scale)[(size_t)r * (K / 128) + c / 128];
                v = q * s;
            } else if (fmt == OF_MXFP4 || fmt == OF_NVFP4) {
                uint8_t byte = ((const uint8_t *)w)[i / 2];
                int code = (c & 1) ? (byte >> 4) : (byte & 15);
                float q = (float)oracle_e2m1(code);
                if (fmt == OF_MXFP4) {
                    if (K % 32) return -1;
                    float s = (float)oracle_e8m0(((const uint8_t *)scale)[(size_t)r * (K / 32) + c / 32]);
                    v = q * s;
                } else {
                    if (K % 16) return -1;
                    float s = (float)oracle_e4m3(((const uint8_t *)scale)[(size_t)r * (K / 16) + c / 16]);
                    v = (q * s) * tscale; /* in this multiplication order */
                }
            } else {
                return -1;
            }
            out[i] = v;
        }
    }
    return 0;
}

/* Bytes of one expert tensor [rows, K] and of its scale plane. */
static size_t tensor_bytes(int fmt, int rows, int K) {
    size_t n = (size_t)rows * K;
    return fmt == OF_BF16 ? 2 * n : fmt == OF_FP8 ? n : n / 2;
}
static size_t scale_bytes(int fmt, int rows, int K) {
    size_t n = (size_t)rows * K;
    return fmt == OF_FP8 ? 4 * (n / 128) : fmt == OF_MXFP4 ? n / 32 : fmt == OF_NVFP4 ? n / 16 : 0;
}

/* --------------------------------------------------- activation format A4 */

/* READING (activation format). Besides the plain form (A16: x as given in bf16,
 * h rounded to bf16), the layer's activations may be carried in the NVFP4 form
 * the aimodeling.com page names among its formats ("Reported Numbers and
 * Ecosystem Position"), so that both operands of every expert GEMM are FP4:
 *   x: one per-tensor scale s_g = amax(|x|) / (6 * 448) over the whole [T, H]
 *      batch (s_g = 1 when every element is 0);
 *   h: s_g = 1 (h is quantised row by row as it is produced);
 *   per 16 consecutive elements along K: s_b = E4M3_RN_sat((amax_b / 6) / s_g);
 *   codes q = E2M1_RNE_sat(v / (s_b * s_g)), 0 where s_b * s_g is 0;
 *   the value the GEMM sees is (q * s_b) * s_g.
 * Every step is one binary32 operation in the order written. E4M3_RN_sat and
 * E2M1_RNE_sat round to the nearest representable value, ties to the even
 * code (mantissa bit 0), and clamp magnitudes beyond the largest value (448,
 * 6) to it. */

/* Nearest E4M3 code of a magnitude v >= 0 (ties to the even code, saturating). */
static int e4m3_rn_sat(float v) {
    if (!(v > 0.0f)) return 0;
    if (v >= 448.0f) return 0x7E;
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(oracle_e4m3(c) - (double)v);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return best;
}

/* Nearest E2M1 code of v (ties to the even code, saturating at 6); bit 3 = sign. */
static int e2m1_rne_sat(float v) {
    int sgn = v < 0.0f ? 8 : 0;
    double a = fabs((double)v);
    if (a >= 6.0) return 7 | sgn;   /* saturate (far beyond 6 the distances would tie in binary64) */
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(oracle_e2m1(c) - a);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return best | sgn;
}

int oracle_e4m3_encode(float v) { return e4m3_rn_sat(v); }
int oracle_e2m1_encode(float v) { return e2m1_rne_sat(v); }

/* Per-tensor scale of x in A4 form: amax(|x|) / (6 * 448), or 1 for an all-zero x. */
float oracle_a4_tensor_scale(const uint16_t *x, size_t n) {
    float amax = 0.0f;
    for (size_t i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(bf16_to_f32(x[i])));
    return amax > 0.0f ? amax / (6.0f * 448.0f) : 1.0f;
}

/* A4 form of v[K] (K a multiple of 16) with tensor scale s_g: out = (q * s_b) * s_g;
 * codes (nullable) get the E2M1 codes, scales (nullable) the E4M3 codes, one per block. */
void oracle_a4_quant(const float *v, int K, float s_g, float *out, uint8_t *codes, uint8_t *scales) {
    for (int b = 0; b < K; b += 16) {
        float amax = 0.0f;
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[b + i]));
        int sc = e4m3_rn_sat((amax / 6.0f) / s_g);
        float sb = (float)oracle_e4m3(sc);
        float den = sb * s_g;
        if (scales) scales[b / 16] = (uint8_t)sc;
        for (int i = 0; i < 16; ++i) {
            int q = den > 0.0f ? e2m1_rne_sat(v[b + i] / den) : 0;
            if (codes) codes[b + i] = (uint8_t)q;
            out[b + i] = ((float)oracle_e2m1(q) * sb) * s_g;
        }
    }
}

/* ---------------------------------------------------------------- router */

/* Router logits, top-k and gating for T tokens.
 * READING (logits): l[t,e] = fl32( sum_h x[t,h]*Wr[h,e] ) with every product and
 *   the running sum in binary64 (bf16*bf16 and bf16*fp32 products are exact in
 *   binary64), rounded once to binary32, then l += bias[e] as one binary32 add.
 * READING (selection): experts ordered by logit descending, ties to the lower
 *   expert index; the first k are chosen. Selection uses logits, not
 *   probabilities, so exp() cannot create ties.
 * READING (gating): softmax over the k selected logits only,
 *   w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), in binary32.
 * wr: [H, E] row-major, fp32 if wr_is_fp32 else bf16 bits. bias nullable [E].
 * Outputs idx [T,k] int32, w [T,k] fp32, logits nullable [T,E] fp32. */
void oracle_route(const uint16_t *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E,
                  int k, int32_t *idx, float *w, float *logits) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        float *l = (float *)malloc(sizeof(float) * E);
        int *order = (int *)malloc(sizeof(int) * E);
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h) {
                double xv = bf16_to_f32(x[(size_t)t * H + h]);
                double wv = wr_is_fp32 ? ((const float *)wr)[(size_t)h * E + e]
                                       : bf16_to_f32(((const uint16_t *)wr)[(size_t)h * E + e]);
                acc += xv * wv;
            }
            float lf = (float)acc;
            if (bias) lf = lf + bias[e];
            l[e] = lf;
            if (logits) logits[(size_t)t * E + e] = lf;
        }
        /* selection: k passes of "largest remaining, lowest index on ties" */
        char *taken = (char *)calloc(E, 1);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            order[j] = best;
        }
        float l0 = l[order[0]], z = 0.0f;
        for (int j = 0; j < k; ++j) z += expf(l[order[j]] - l0);
        for (int j = 0; j < k; ++j) {
            idx[(size_t)t * k + j] = order[j];
            w[(size_t)t * k + j] = expf(l[order[j]] - l0) / z;
        }
        free(taken);
        free(l);
        free(order);
    }
}

/* ----------------------------------------------------------- permutation */

/* Token-to-expert permutation (counting sort, stable in the pair index).
 * A pair is p = t*k + j. counts[e] = #pairs routed to e; offsets = exclusive
 * scan of counts, offsets[E] = T*k. Within an expert, pairs keep ascending p:
 * sorted_pair[offsets[e] + r] is the r-th such p, pair_row[p] its row. */
void oracle_permute(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *sorted_pair,
                    int32_t *pair_row) {
    int P = T * k;
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int p = 0; p < P; ++p) offsets[idx[p] + 1] += 1;
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    int *fill = (int *)calloc((size_t)(E > 0 ? E : 1), sizeof(int));
    for (int p = 0; p < P; ++p) {
        int e = idx[p];
        int r = offsets[e] + fill[e]++;
        sorted_pair[r] = p;
        pair_row[p] = r;
    }
    free(fill);
}

/* -------------------------------------------------------------------- FFN */

static float silu(float z) { return z / (1.0f + expf(-z)); }

/* SwiGLU expert FFN for the rows of one expert, weights already dequantised.
 * For each row: g = x.Wg^T, u = x.Wu^T (binary32, sequential in h);
 * h = silu(g)*u with silu(z) = z/(1+exp(-z));
 * READING: h is rounded to bf16 (to nearest even) before the down projection;
 * y = h.W2^T in binary32. w13f [2I, H] (gate rows then up rows), w2f [H, I]. */
static void ffn_rows(const uint16_t *x, const int32_t *tok_of_row, int nrows, int H, int I, const float *w13f,
                     const float *w2f, float *hbuf, float *y, float *h_out, int act, float s_gx) {
    float *xr = (float *)malloc(sizeof(float) * H);
    for (int r = 0; r < nrows; ++r) {
        int t = tok_of_row[r];
        for (int c = 0; c < H; ++c) xr[c] = bf16_to_f32(x[(size_t)t * H + c]);
        if (act == ACT_A4) oracle_a4_quant(xr, H, s_gx, xr, 0, 0);   /* READING: activation format A4 */
        for (int i = 0; i < I; ++i) {
            float g = 0.0f, u = 0.0f;
            const float *wg = w13f + (size_t)i * H, *wu = w13f + (size_t)(I + i) * H;
            for (int c = 0; c < H; ++c) g += xr[c] * wg[c];
            for (int c = 0; c < H; ++c) u += xr[c] * wu[c];
            float hv = bf16_to_f32(f32_to_bf16(silu(g) * u));
            if (act == ACT_A4) hv = silu(g) * u;   /* quantised below, with the whole row */
            hbuf[i] = hv;
            if (h_out) h_out[(size_t)r * I + i] = hv;
        }
        if (act == ACT_A4) {
            oracle_a4_quant(hbuf, I, 1.0f, hbuf, 0, 0);
            if (h_out) memcpy(h_out + (size_t)r * I, hbuf, sizeof(float) * I);
        }
        for (int j = 0; j < H; ++j) {
            float acc = 0.0f;
            const float *w2r = w2f + (size_t)j * I;
            for (int i = 0; i < I; ++i) acc += hbuf[i] * w2r[i];
            y[(size_t)r * H + j] = acc;
        }
    }
    free(xr);
}

/* Expert FFN over the permuted pairs of all experts that received any.
 * w13/w2 (+ scales, tscales) are dense [E][...] arrays in the stored formats.
 * Writes y_perm [T*k, H] fp32 and, if h_out is non-null, h [T*k, I] (bf16 values in fp32).
 * Returns 0, or -1 on a bad format. */
int oracle_ffn(const uint16_t *x, int T, int H, int I, int E, int k, int fmt, const void *w13, const void *w13s,
               const float *w13t, const void *w2, const void *w2s, const float *w2t, const int32_t *offsets,
               const int32_t *sorted_pair, float *y_perm, float *h_out, int act) {
    size_t b13 = tensor_bytes(fmt, 2 * I, H), s13 = scale_bytes(fmt, 2 * I, H);
    size_t b2 = tensor_bytes(fmt, H, I), s2 = scale_bytes(fmt, H, I);
    float s_gx = act == ACT_A4 ? oracle_a4_tensor_scale(x, (size_t)T * H) : 1.0f;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int e = 0; e < E; ++e) {
        int n = offsets[e + 1] - offsets[e];
        if (n == 0) continue;
        float *w13f = (float *)malloc(sizeof(float) * (size_t)2 * I * H);
        float *w2f = (float *)malloc(sizeof(float) * (size_t)H * I);
        float *hbuf = (float *)malloc(sizeof(float) * I);
        int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * n);
        bad |= oracle_dequant(fmt, 2 * I, H, (const char *)w13 + e * b13, w13s ? (const char *)w13s + e * s13 : 0,
                              w13t ? w13t[e] : 1.0f, w13f) != 0;
        bad |= oracle_dequant(fmt, H, I, (const char *)w2 + e * b2, w2s ? (const char *)w2s + e * s2 : 0,
                              w2t ? w2t[e] : 1.0f, w2f) != 0;
        for (int r = 0; r < n; ++r) tok[r] = sorted_pair[offsets[e] + r] / k;
        ffn_rows(x, tok, n, H, I, w13f, w2f, hbuf, y_perm + (size_t)offsets[e] * H,
                 h_out ? h_out + (size_t)offsets[e] * I : 0, act, s_gx);
        free(w13f);
        free(w2f);
        free(hbuf);
        free(tok);
    }
    return bad ? -1 : 0;
}

/* ---------------------------------------------------------------- combine */

/* Gate-weighted combine: out[t] = sum_{j=0..k-1} w[t,j] * y_perm[pair_row[t*k+j]],
 * accumulated in binary32 in order of j. out is [T, H] fp32. */
void oracle_combine(const float *y_perm, const int32_t *pair_row, const float *w, int T, int k, int H, float *out) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int r = pair_row[(size_t)t * k + j];
                acc += w[(size_t)t * k + j] * y_perm[(size_t)r * H + c];
            }
            out[(size_t)t * H + c] = acc;
        }
    }
}

/* ------------------------------------------------------------ whole layer */

/* The whole layer: route -> permute -> FFN -> combine. Scratch is allocated here.
 * Any output pointer except out may be null. Returns 0 or -1. */
int oracle_layer(const uint16_t *x, int T, int H, const void *wr, int wr_is_fp32, const float *bias, int E, int k,
                 int I, int fmt, const void *w13, const void *w13s, const float *w13t, const void *w2,
                 const void *w2s, const float *w2t, int32_t *idx_out, float *w_out, int32_t *offsets_out,
                 int32_t *sorted_out, int32_t *pair_row_out, float *y_perm_out, float *out, int act) {
    int P = T * k;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (P ? P : 1));
    float *w = (float *)malloc(sizeof(float) * (P ? P : 1));
    int32_t *off = (int32_t *)malloc(sizeof(int32_t) * (E + 1));
    int32_t *sp = (int32_t *)malloc(sizeof(int32_t) * (P ? P : 1));
    int32_t *pr = (int32_t *)malloc(sizeof(int32_t) * (P ? P : 1));
    float *y = (float *)malloc(sizeof(float) * (size_t)(P ? P : 1) * H);
    oracle_route(x, T, H, wr, wr_is_fp32, bias, E, k, idx, w, 0);
    oracle_permute(idx, T, k, E, off, sp, pr);
    int rc = oracle_ffn(x, T, H, I, E, k, fmt, w13, w13s, w13t, w2, w2s, w2t, off, sp, y, 0, act);
    oracle_combine(y, pr, w, T, k, H, out);
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * P);
    if (w_out) memcpy(w_out, w, sizeof(float) * P);
    if (offsets_out) memcpy(offsets_out, off, sizeof(int32_t) * (E + 1));
    if (sorted_out) memcpy(sorted_out, sp, sizeof(int32_t) * P);
    if (pair_row_out) memcpy(pair_row_out, pr, sizeof(int32_t) * P);
    if (y_perm_out) memcpy(y_perm_out, y, sizeof(float) * (size_t)P * H);
    free(idx);
    free(w);
    free(off);
    free(sp);
    free(pr);
    free(y);
    return rc;
}

/* Output rows of selected tokens only, given the routing (idx, w) of the full
 * batch: out_rows[i] = sum_j w[t,j] * FFN_{idx[t,j]}(x[t]) for t = tokens[i].
 * Weights are dequantised per (token, expert) on the fly, so the cost is
 * independent of T. Used to check full-size runs on sampled outputs. */
int oracle_token_rows(const uint16_t *x, int H, int I, int k, int fmt, const void *w13, const void *w13s,
                      const float *w13t, const void *w2, const void *w2s, const float *w2t, const int32_t *idx,
                      const float *w, const int32_t *tokens, int ntok, float *out_rows, int T, int act) {
    size_t b13 = tensor_bytes(fmt, 2 * I, H), s13 = scale_bytes(fmt, 2 * I, H);
    size_t b2 = tensor_bytes(fmt, H, I), s2 = scale_bytes(fmt, H, I);
    float s_gx = act == ACT_A4 ? oracle_a4_tensor_scale(x, (size_t)T * H) : 1.0f;   /* over the whole batch */
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int i = 0; i < ntok; ++i) {
        int t = tokens[i];
        float *w13f = (float *)malloc(sizeof(float) * (size_t)2 * I * H);
        float *w2f = (float *)malloc(sizeof(float) * (size_t)H * I);
        float *hbuf = (float *)malloc(sizeof(float) * I);
        float *y = (float *)malloc(sizeof(float) * H);
        float *acc = out_rows + (size_t)i * H;
        for (int c = 0; c < H; ++c) acc[c] = 0.0f;
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            bad |= oracle_dequant(fmt, 2 * I, H, (const char *)w13 + e * b13, w13s ? (const char *)w13s + e * s13 : 0,
                                  w13t ? w13t[e] : 1.0f, w13f) != 0;
            bad |= oracle_dequant(fmt, H, I, (const char *)w2 + e * b2, w2s ? (const char *)w2s + e * s2 : 0,
                                  w2t ? w2t[e] : 1.0f, w2f) != 0;
            int32_t tok = t;
            ffn_rows(x, &tok, 1, H, I, w13f, w2f, hbuf, y, 0, act, s_gx);
            for (int c = 0; c < H; ++c) acc[c] += w[(size_t)t * k + j] * y[c];
        }
        free(w13f);
        free(w2f);
        free(hbuf);
        free(y);
    }
    return bad ? -1 : 0;
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
