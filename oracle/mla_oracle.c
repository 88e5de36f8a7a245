/*
 * mla_oracle.c -- plain, slow, float64 CPU oracle for Multi-head Latent Attention (MLA).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg call this file.  It shares no code, header or table with the CUDA library.
 *
 * Every function is written as the definition it follows, one loop per sum, accumulating
 * in double, with no blocking, fusion or reordering.  Sources (page title, section):
 *
 *  [L1] "02 - Multi-Latent Attention (MLA)" (lynx-cortex course, phase 36):
 *       "Multi-head attention estandar" (q = W_Q h), "La compresion de MLA"
 *       (c_t = W_DKV h_t; k_t = W_UK c_t, v_t = W_UV c_t), "Truco de codificacion
 *       posicional" (a decoupled rotary key k^rope of width d_hR is cached as is),
 *       "Coste de computo" (the up-projections can be absorbed so that attention runs
 *       on c directly), "Lo que MLA no es" (the reconstructed K and V are exactly
 *       W_UK c and W_UV c: absorption is not an approximation).
 *  [L2] "Multi-head latent attention" (aiunderstanding.org), "Informacion tecnica":
 *       up-projections absorbed into the query and output projections; RoPE handled by
 *       a separate decoupled key path.
 *  [L4] "Multi-head Latent Attention (MLA) si arhitectura DeepSeekMoE" (dexblog.ro),
 *       opening section: the cache keeps only the latent and a small decoupled RoPE
 *       key, (d_c + d_hR) elements per token per layer.
 *  [L5] "DeepSeek MLA" (llm-engineer cards), section on the RoPE problem:
 *       attention score = content score + positional score.
 *
 * Readings where the pages are silent (each one shared by both sides of a parity test):
 *  - RoPE: interleaved pairs (2i, 2i+1) rotated by pos * theta^(-2i/d), theta = 10000;
 *    one rotary key per token, shared by all heads.
 *  - softmax scale 1/sqrt(qk_nope + d_hR); the query attends to every row it is given.
 *  - W_Q rows are head-major, qk_nope content rows then d_hR rotary rows per head.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ sizes [L1][L4] */

/* Elements one token adds to a standard multi-head KV cache per layer: k and v. [L1] */
int64_t oracle_mha_elems_per_token(int64_t n_heads, int64_t d_head) {
    return 2 * n_heads * d_head;
}

/* Elements one token adds to the MLA cache over `layers` layers: (d_c + d_hR) * l. [L4] */
int64_t oracle_mla_elems_per_token(int64_t d_c, int64_t d_hR, int64_t layers) {
    return (d_c + d_hR) * layers;
}

/* ------------------------------------------------------------- rounding helpers */

/* float64 -> bfloat16 bits, round to nearest, ties to even, in one step (no float32 stop). */
uint16_t oracle_round_bf16(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    if (a == 0.0) return sign;
    int e;
    double m = frexp(a, &e);               /* a = m * 2^e, m in [0.5, 1) */
    if (e - 1 < -126) {                    /* subnormal: quantum 2^-133 */
        double r = rint(ldexp(a, 133));    /* rint: ties to even in the default mode */
        return (uint16_t)(sign | (uint16_t)r);   /* r == 128 carries into the exponent */
    }
    double r = rint(ldexp(m, 8));          /* 8 significant bits, in [128, 256] */
    if (r == 256.0) { r = 128.0; e += 1; }
    int be = e - 1 + 127;
    if (be >= 255) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | (uint16_t)(be << 7) | (uint16_t)((int)r - 128));
}

void oracle_round_bf16_array(int64_t n, const double* x, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

/* float64 -> the value of the nearest FP8 E4M3 number (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, largest finite 448, subnormals down to 2^-9), ties to even.
 * Magnitudes above 448 saturate to 448 (the per-token scale below never produces them). */
double oracle_round_e4m3(double x) {
    double a = fabs(x);
    if (isnan(x)) return x;
    if (a == 0.0) return x;
    int e;
    frexp(a, &e);                          /* a = m * 2^e, m in [0.5, 1): exponent e - 1 */
    int ue = e - 1 < -6 ? -6 : e - 1;      /* below 2^-6 the quantum stays 2^-9 */
    double q = ldexp(1.0, ue - 3);         /* 3 mantissa bits */
    double r = rint(a / q) * q;            /* rint: ties to even in the default mode */
    if (r > 448.0) r = 448.0;
    return signbit(x) ? -r : r;
}

/* -------------------------------------------------- FP8 latent cache [L1][L4] */

/* A quantised latent cache, which [L1] ("Lo que esta fase NO cubre": quantised KV cache as
 * another compression) and [L4] ("Exemplul 1": the engine's real cache format, e.g. FP8)
 * name without a format.  Reading: each token's latent c (d_c values) is stored as FP8 E4M3
 * codes with one scale per token, s = max_i |c_i| / 448 (s = 1 for an all-zero c), code_i =
 * e4m3(c_i / s); the decoupled RoPE key stays as it is.  The attention then runs on the
 * dequantised row [code * s | k_r].  rows, deq: [n, d_c + d_hR]; scales: [n]. */
void oracle_quantize_latent_fp8(int n, int d_c, int d_hR, const double* rows, double* deq,
                                double* scales) {
    int rw = d_c + d_hR;
    for (int t = 0; t < n; ++t) {
        const double* r = rows + (size_t)t * rw;
        double* o = deq + (size_t)t * rw;
        double amax = 0.0;
        for (int i = 0; i < d_c; ++i) amax = fmax(amax, fabs(r[i]));
        double sc = amax > 0.0 ? amax / 448.0 : 1.0;
        for (int i = 0; i < d_c; ++i) o[i] = oracle_round_e4m3(r[i] / sc) * sc;
        for (int i = 0; i < d_hR; ++i) o[d_c + i] = r[d_c + i];
        scales[t] = sc;
    }
}

/* The E4M3 bit pattern of a value that round_e4m3 returns: sign in bit 7, the exponent field
 * (bias 7; 0 for subnormals) in bits 6-3, the 3 mantissa bits in 2-0.  448 = 1.75 * 2^8 is
 * 0x7E; the pattern 0x7F (NaN) never comes out. */
uint8_t oracle_e4m3_bits(double v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    double m = frexp(a, &e);               /* a = m * 2^e, m in [0.5, 1) */
    int ex = e - 1;                        /* a = (2m) * 2^ex, 2m in [1, 2) */
    if (ex < -6) {                         /* subnormal: a = k * 2^-9, k in 1 .. 7 */
        int k = (int)rint(ldexp(a, 9));
        return (uint8_t)(sign | k);
    }
    int mant = (int)rint((2.0 * m - 1.0) * 8.0);
    return (uint8_t)(sign | ((ex + 7) << 3) | mant);
}

/* The FP8 cache row a kernel writes for one bf16 row [c | k_r] (d_c latent values, d_hR
 * rotary values, both exactly representable in float), with every rounding decision taken
 * in float (IEEE single, nearest even), as a kernel working in fp32 takes it:
 *     amax = max |c_i|,  s = amax / 448 (s = 1 for amax = 0),  code_i = e4m3(c_i / s).
 * Writes row_bytes bytes: the d_c codes, the d_hR rotary values as bf16 (the top 16 bits
 * of their float patterns, exact for bf16 inputs), s as a float, zeros up to row_bytes.
 * deq (nullable, d_c + d_hR doubles) receives [code_i * s | k_r]. */
void oracle_fp8_row_f32(int d_c, int d_hR, const double* row, int row_bytes, uint8_t* out, double* deq) {
    float amax = 0.0f;
    for (int i = 0; i < d_c; ++i) {
        float a = fabsf((float)row[i]);
        if (a > amax) amax = a;
    }
    volatile float num = amax, den = 448.0f;   /* one float division, not folded */
    float s = amax > 0.0f ? num / den : 1.0f;
    memset(out, 0, (size_t)row_bytes);
    for (int i = 0; i < d_c; ++i) {
        volatile float ci = (float)row[i];
        float q = ci / s;
        double code = oracle_round_e4m3((double)q);
        out[i] = oracle_e4m3_bits(code);
        if (deq) deq[i] = code * (double)s;
    }
    for (int i = 0; i < d_hR; ++i) {
        float v = (float)row[d_c + i];
        uint32_t bits;
        memcpy(&bits, &v, 4);
        uint16_t b = (uint16_t)(bits >> 16);
        memcpy(out + d_c + 2 * i, &b, 2);
        if (deq) deq[d_c + i] = row[d_c + i];
    }
    memcpy(out + d_c + 2 * d_hR, &s, 4);
}

/* ------------------------------------------------------------------- RoPE [L1][L2] */

/* out = x rotated: for i < d/2, angle = pos * theta^(-2i/d),
 * (out[2i], out[2i+1]) = (x[2i] cos - x[2i+1] sin, x[2i] sin + x[2i+1] cos). */
void oracle_rope(int d, const double* x, double pos, double theta, double* out) {
    for (int i = 0; i < d / 2; ++i) {
        double ang = pos * pow(theta, -2.0 * (double)i / (double)d);
        double c = cos(ang), s = sin(ang);
        double x0 = x[2 * i], x1 = x[2 * i + 1];
        out[2 * i] = x0 * c - x1 * s;
        out[2 * i + 1] = x0 * s + x1 * c;
    }
}

/* The rotation of RoPE pairs restated in the precision kernels rotate in: for pair i, with
 * (c, s) = cs[2i], cs[2i+1],
 *     y[2i] = float(x0 c - x1 s),   y[2i+1] = float(x0 s + x1 c)
 * in IEEE double, each product and sum rounded on its own (this file is compiled without
 * contraction into fused multiply-adds), then rounded to float once. */
void oracle_rope_pairs_f32(int64_t pairs, const float* x, const double* cs, float* y) {
    for (int64_t i = 0; i < pairs; ++i) {
        double x0 = x[2 * i], x1 = x[2 * i + 1], c = cs[2 * i], s = cs[2 * i + 1];
        double p0 = x0 * c, p1 = x1 * s, p2 = x0 * s, p3 = x1 * c;
        y[2 * i] = (float)(p0 - p1);
        y[2 * i + 1] = (float)(p2 + p3);
    }
}

/* ------------------------------------------------- latent cache rows [L1][L4][L5] */

/* For each token i: c = W_DKV h_i (d_c values), k_r = RoPE(W_KR h_i, pos_i) (d_hR values);
 * the cache row is [c | k_r], d_c + d_hR wide.  h: [n, d_model]; W_DKV: [d_c, d_model];
 * W_KR: [d_hR, d_model]; rows: [n, d_c + d_hR]. */
void oracle_latent_rows(int n, int d_model, int d_c, int d_hR, const double* h,
                        const double* W_DKV, const double* W_KR, const int32_t* pos,
                        double theta, double* rows) {
    double* kr = (double*)malloc(sizeof(double) * (size_t)d_hR);
    for (int i = 0; i < n; ++i) {
        const double* hi = h + (size_t)i * d_model;
        double* row = rows + (size_t)i * (d_c + d_hR);
        for (int j = 0; j < d_c; ++j) {
            double acc = 0.0;
            for (int k = 0; k < d_model; ++k) acc += W_DKV[(size_t)j * d_model + k] * hi[k];
            row[j] = acc;
        }
        for (int j = 0; j < d_hR; ++j) {
            double acc = 0.0;
            for (int k = 0; k < d_model; ++k) acc += W_KR[(size_t)j * d_model + k] * hi[k];
            kr[j] = acc;
        }
        oracle_rope(d_hR, kr, (double)pos[i], theta, row + d_c);
    }
    free(kr);
}

/* ------------------------------------------------------------ query [L1][L2] */

/* q = W_Q h (standard projection); per head, the first qk_nope values are the content
 * query, the last d_hR values are rotated at the token's position.
 * h: [n, d_model]; W_Q: [H*(qk_nope+d_hR), d_model]; q_nope: [n, H, qk_nope];
 * q_rope: [n, H, d_hR]. */
void oracle_query(int n, int d_model, int H, int qk_nope, int d_hR, const double* h,
                  const double* W_Q, const int32_t* pos, double theta, double* q_nope,
                  double* q_rope) {
    int qh = qk_nope + d_hR;
    double* q = (double*)malloc(sizeof(double) * (size_t)qh);
    for (int i = 0; i < n; ++i) {
        const double* hi = h + (size_t)i * d_model;
        for (int hd = 0; hd < H; ++hd) {
            for (int j = 0; j < qh; ++j) {
                const double* w = W_Q + ((size_t)hd * qh + j) * d_model;
                double acc = 0.0;
                for (int k = 0; k < d_model; ++k) acc += w[k] * hi[k];
                q[j] = acc;
            }
            memcpy(q_nope + ((size_t)i * H + hd) * qk_nope, q, sizeof(double) * qk_nope);
            oracle_rope(d_hR, q + qk_nope, (double)pos[i], theta,
                        q_rope + ((size_t)i * H + hd) * d_hR);
        }
    }
    free(q);
}

/* ------------------------------------------------------------------ softmax */

/* p = softmax(s) over T scores (max subtracted first); returns log-sum-exp of s.
 * An empty row (T = 0) has no probabilities; its log-sum-exp is -inf and the attention
 * output over it is taken as zero. */
static double softmax_inplace(int T, double* s) {
    if (T <= 0) return -INFINITY;
    double m = -INFINITY;
    for (int t = 0; t < T; ++t) if (s[t] > m) m = s[t];
    double l = 0.0;
    for (int t = 0; t < T; ++t) { s[t] = exp(s[t] - m); l += s[t]; }
    for (int t = 0; t < T; ++t) s[t] /= l;
    return m + log(l);
}

/* --------------------------------------------- one decode head, naive [L1][L5] */

/* One query of one head attending over T cache rows, with K and V materialised:
 *   k_nope[t] = W_UK_h c_t (qk_nope), v[t] = W_UV_h c_t (v_head),
 *   s[t] = scale * (q_nope . k_nope[t] + q_rope . k_r,t),  p = softmax(s),
 *   o = sum_t p[t] v[t].
 * rows: [T, d_c + d_hR] = [c | k_r]; W_UK_h: [qk_nope, d_c]; W_UV_h: [v_head, d_c].
 * p_out (nullable) receives p; lse_out (nullable) receives log sum_t exp(s[t]). */
void oracle_attend_naive(int T, int d_c, int d_hR, int qk_nope, int v_head, double scale,
                         const double* q_nope, const double* q_rope, const double* rows,
                         const double* W_UK_h, const double* W_UV_h, double* o,
                         double* p_out, double* lse_out) {
    int rw = d_c + d_hR;
    double* s = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double* k = (double*)malloc(sizeof(double) * (size_t)qk_nope);
    double* v = (double*)malloc(sizeof(double) * (size_t)v_head);
    for (int t = 0; t < T; ++t) {
        const double* c = rows + (size_t)t * rw;
        for (int j = 0; j < qk_nope; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d_c; ++i) acc += W_UK_h[(size_t)j * d_c + i] * c[i];
            k[j] = acc;
        }
        double content = 0.0, positional = 0.0;
        for (int j = 0; j < qk_nope; ++j) content += q_nope[j] * k[j];
        for (int j = 0; j < d_hR; ++j) positional += q_rope[j] * c[d_c + j];
        s[t] = scale * (content + positional);
    }
    double lse = softmax_inplace(T, s);
    for (int j = 0; j < v_head; ++j) o[j] = 0.0;
    for (int t = 0; t < T; ++t) {
        const double* c = rows + (size_t)t * rw;
        for (int j = 0; j < v_head; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d_c; ++i) acc += W_UV_h[(size_t)j * d_c + i] * c[i];
            v[j] = acc;
        }
        for (int j = 0; j < v_head; ++j) o[j] += s[t] * v[j];
    }
    if (p_out) memcpy(p_out, s, sizeof(double) * (size_t)T);
    if (lse_out) *lse_out = lse;
    free(s); free(k); free(v);
}

/* ---------------------------------------- one decode head, absorbed [L1][L2][L4] */

/* The same result with the up-projections absorbed:
 *   q_lat = W_UK_h^T q_nope (d_c), s[t] = scale * (q_lat . c_t + q_rope . k_r,t),
 *   p = softmax(s), o_lat = sum_t p[t] c_t (d_c), o = W_UV_h o_lat. */
void oracle_attend_absorbed(int T, int d_c, int d_hR, int qk_nope, int v_head, double scale,
                            const double* q_nope, const double* q_rope, const double* rows,
                            const double* W_UK_h, const double* W_UV_h, double* o,
                            double* p_out, double* lse_out) {
    int rw = d_c + d_hR;
    double* s = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double* q_lat = (double*)malloc(sizeof(double) * (size_t)d_c);
    double* o_lat = (double*)malloc(sizeof(double) * (size_t)d_c);
    for (int i = 0; i < d_c; ++i) {
        double acc = 0.0;
        for (int j = 0; j < qk_nope; ++j) acc += W_UK_h[(size_t)j * d_c + i] * q_nope[j];
        q_lat[i] = acc;
    }
    for (int t = 0; t < T; ++t) {
        const double* c = rows + (size_t)t * rw;
        double content = 0.0, positional = 0.0;
        for (int i = 0; i < d_c; ++i) content += q_lat[i] * c[i];
        for (int j = 0; j < d_hR; ++j) positional += q_rope[j] * c[d_c + j];
        s[t] = scale * (content + positional);
    }
    double lse = softmax_inplace(T, s);
    for (int i = 0; i < d_c; ++i) o_lat[i] = 0.0;
    for (int t = 0; t < T; ++t) {
        const double* c = rows + (size_t)t * rw;
        for (int i = 0; i < d_c; ++i) o_lat[i] += s[t] * c[i];
    }
    for (int j = 0; j < v_head; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d_c; ++i) acc += W_UV_h[(size_t)j * d_c + i] * o_lat[i];
        o[j] = acc;
    }
    if (p_out) memcpy(p_out, s, sizeof(double) * (size_t)T);
    if (lse_out) *lse_out = lse;
    free(s); free(q_lat); free(o_lat);
}

/* ------------------------------------------------------------ decode batch driver */

/* Decode for a list of (sequence b, head h) units.  Sequence b owns rows
 * [offsets[b], offsets[b+1]) of `rows`.  q_nope: [B, H, qk_nope]; q_rope: [B, H, d_hR];
 * W_UK: [H, qk_nope, d_c]; W_UV: [H, v_head, d_c]; o: [n_units, v_head];
 * lse (nullable): [n_units].  absorbed = 0 runs the naive form, 1 the absorbed form. */
void oracle_decode(int absorbed, int H, int d_c, int d_hR, int qk_nope, int v_head,
                   double scale, const int64_t* offsets, const double* q_nope,
                   const double* q_rope, const double* rows, const double* W_UK,
                   const double* W_UV, int n_units, const int32_t* unit_b,
                   const int32_t* unit_h, double* o, double* lse) {
    int rw = d_c + d_hR;
    for (int u = 0; u < n_units; ++u) {
        int b = unit_b[u], h = unit_h[u];
        int64_t t0 = offsets[b], T = offsets[b + 1] - offsets[b];
        const double* qn = q_nope + ((size_t)b * H + h) * qk_nope;
        const double* qr = q_rope + ((size_t)b * H + h) * d_hR;
        const double* wk = W_UK + (size_t)h * qk_nope * d_c;
        const double* wv = W_UV + (size_t)h * v_head * d_c;
        double* ou = o + (size_t)u * v_head;
        double* lu = lse ? lse + u : NULL;
        if (absorbed)
            oracle_attend_absorbed((int)T, d_c, d_hR, qk_nope, v_head, scale, qn, qr,
                                   rows + (size_t)t0 * rw, wk, wv, ou, NULL, lu);
        else
            oracle_attend_naive((int)T, d_c, d_hR, qk_nope, v_head, scale, qn, qr,
                                rows + (size_t)t0 * rw, wk, wv, ou, NULL, lu);
    }
}

/* ------------------------------------------------- multi-token decode [L4][L1] */

/* Several new tokens per sequence in one step: the verification of draft tokens in
 * speculative decoding, which [L4] ("Concepte cheie": the MTP module) names as a use of
 * multi-token prediction.  The pages give no formula; the reading taken is the causal rule
 * of attention within the sequence ([L1] "La compresion de MLA": each token attends to the
 * tokens before it and itself).  Sequence b owns rows [offsets[b], offsets[b+1]); its last
 * q_len rows are the new tokens.  New token t (0 <= t < q_len) sits at position
 * L_b - q_len + t and attends to rows 0 .. L_b - q_len + t of its sequence.
 * Units are (b, t, h).  q_nope: [B, q_len, H, qk_nope]; q_rope: [B, q_len, H, d_hR];
 * o: [n_units, v_head].  A token with no rows (L_b - q_len + t < 0) gives o = 0. */
void oracle_decode_multi(int absorbed, int H, int q_len, int d_c, int d_hR, int qk_nope, int v_head,
                         double scale, const int64_t* offsets, const double* q_nope,
                         const double* q_rope, const double* rows, const double* W_UK,
                         const double* W_UV, int n_units, const int32_t* unit_b,
                         const int32_t* unit_t, const int32_t* unit_h, double* o) {
    int rw = d_c + d_hR;
    for (int u = 0; u < n_units; ++u) {
        int b = unit_b[u], t = unit_t[u], h = unit_h[u];
        int64_t t0 = offsets[b];
        int64_t T = offsets[b + 1] - offsets[b] - (q_len - 1 - t);   /* keys up to the token itself */
        if (T < 0) T = 0;
        size_t q = ((size_t)b * q_len + t) * H + h;
        const double* wk = W_UK + (size_t)h * qk_nope * d_c;
        const double* wv = W_UV + (size_t)h * v_head * d_c;
        double* ou = o + (size_t)u * v_head;
        if (absorbed)
            oracle_attend_absorbed((int)T, d_c, d_hR, qk_nope, v_head, scale, q_nope + q * qk_nope,
                                   q_rope + q * d_hR, rows + (size_t)t0 * rw, wk, wv, ou, NULL, NULL);
        else
            oracle_attend_naive((int)T, d_c, d_hR, qk_nope, v_head, scale, q_nope + q * qk_nope,
                                q_rope + q * d_hR, rows + (size_t)t0 * rw, wk, wv, ou, NULL, NULL);
    }
}

/* ----------------------------------------------------- output projection [L1][L2] */

/* out[i] = W_O concat_h o[i, h, :].  o: [n, H*v_head]; W_O: [d_model, H*v_head]. */
void oracle_out_proj(int n, int Hv, int d_model, const double* o, const double* W_O,
                     double* out) {
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < d_model; ++j) {
            double acc = 0.0;
            for (int k = 0; k < Hv; ++k) acc += W_O[(size_t)j * Hv + k] * o[(size_t)i * Hv + k];
            out[(size_t)i * d_model + j] = acc;
        }
}

/* ------------------------------------------- causal prefill, materialised [L1][L5] */

/* One head of causal self-attention over a sequence of S tokens, K and V materialised
 * from the cache rows: K_t = [W_UK_h c_t | k_r,t], V_t = W_UV_h c_t.  For each query
 * position t in t_list: s[tau] = scale * (q_nope[t] . W_UK_h c_tau + q_rope[t] . k_r,tau)
 * for tau <= t, p = softmax(s), o = sum_tau p[tau] V_tau.
 * q_nope: [S, qk_nope]; q_rope: [S, d_hR] (rotated); rows: [S, d_c+d_hR];
 * o: [n_t, v_head].  absorbed = 1 evaluates the same sums in the absorbed form. */
void oracle_prefill_head(int absorbed, int S, int d_c, int d_hR, int qk_nope, int v_head,
                         double scale, const double* q_nope, const double* q_rope,
                         const double* rows, const double* W_UK_h, const double* W_UV_h,
                         int n_t, const int32_t* t_list, double* o) {
    (void)S;
    for (int u = 0; u < n_t; ++u) {
        int t = t_list[u];
        if (absorbed)
            oracle_attend_absorbed(t + 1, d_c, d_hR, qk_nope, v_head, scale,
                                   q_nope + (size_t)t * qk_nope, q_rope + (size_t)t * d_hR,
                                   rows, W_UK_h, W_UV_h, o + (size_t)u * v_head, NULL, NULL);
        else
            oracle_attend_naive(t + 1, d_c, d_hR, qk_nope, v_head, scale,
                                q_nope + (size_t)t * qk_nope, q_rope + (size_t)t * d_hR, rows,
                                W_UK_h, W_UV_h, o + (size_t)u * v_head, NULL, NULL);
    }
}

/* Softmax probabilities of one naive decode head (used by the probability pins). */
void oracle_attend_probs(int T, int d_c, int d_hR, int qk_nope, int v_head, double scale,
                         const double* q_nope, const double* q_rope, const double* rows,
                         const double* W_UK_h, const double* W_UV_h, double* o,
                         double* p_out) {
    oracle_attend_naive(T, d_c, d_hR, qk_nope, v_head, scale, q_nope, q_rope, rows, W_UK_h,
                        W_UV_h, o, p_out, NULL);
}
