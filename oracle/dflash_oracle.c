/*
 * dflash_oracle.c -- plain, slow fp64 CPU oracle of the DFlash draft-and-verify
 * decode step.  TEST INFRASTRUCTURE ONLY (see dflash_oracle.h): the product
 * library never includes, links or calls this file.
 *
 * What the method computes, as the pages state it:
 *  - a drafter proposes a whole block of tokens in ONE forward pass and the
 *    target checks the whole block in ONE parallel pass ([P2] "O que o DFlash
 *    faz de diferente"; [P4] "Como o DFlash troca o drafter por difusão de
 *    blocos"); 16 tokens per pass ([P5]), 15 speculative ([P2] "Como usar");
 *  - accepted tokens are kept and the output stays identical to target-only
 *    decoding ([P2] "Decodificação especulativa tradicional": lossless;
 *    "6,08x ... temperatura 0"); wrong entries are discarded ([P1]);
 *  - hidden states of several target layers are fused into a compact context
 *    vector that is injected into the Key and Value projections of every
 *    drafter layer and persists in the drafter's KV cache ([P2] "O alvo sabe
 *    mais"; [P4] "Os três mecanismos por trás do DFlash"; [P5]).
 *
 * Readings taken where the pages are silent (each is one plain choice):
 *  R1 decoder layer = pre-norm Llama/Qwen block: x += Wo Attn(RoPE(Wq n),
 *     RoPE(Wk n), Wv n), n = RMSNorm(x); x += Wdown(SiLU(Wgate m) * Wup m),
 *     m = RMSNorm(x).  No biases.  GQA: q head h reads kv head h/(nq/nkv).
 *     Softmax scale 1/sqrt(hd).  RoPE pairs (i, i+hd/2), frequency
 *     theta^(-2i/hd), angle = position * frequency.
 *  R2 target logits = lm_head . RMSNorm_final(x); greedy = argmax, lowest
 *     index on exact ties.
 *  R3 the tapped hidden state of layer l is the residual stream after layer l.
 *  R4 fuse: c = RMSNorm(W_fc . concat(taps in tap order)), eps = drafter eps.
 *  R5 drafter layer j attends over keys/values [RoPE_t(Wk_j c_t), Wv_j c_t]
 *     for every committed position t < p, followed by its own block keys at
 *     p..p+B-1; every block query sees every key (block-bidirectional).  The
 *     context vector is not passed through the layer's input norm.
 *  R6 drafter block = [anchor, mask x (B-1)], embedded with the target's
 *     table; drafter output = its own final norm + the target's lm_head;
 *     drafts = argmax at block rows 1..B-1.
 *  R7 accept: a = largest k <= B-1 with d_i == g_(i-1) for all i <= k;
 *     commit d_1..d_a and the bonus g_a; tau = a+1 tokens per iteration.
 *  R8 MoE FFN: r = softmax(W_r m) over experts; top-k by value (lowest index
 *     on ties); weights renormalised over the chosen k; output = sum of
 *     weighted expert SwiGLUs, in selection order.
 *  R9 no EOS: a generation stops after exactly max_new tokens.
 *
 * Row independence: every per-row reduction (dot products, norms, softmax
 * over keys in position order) is the same code whether one row or a block
 * of rows is processed, so draft-and-verify output equals target-only output
 * bit for bit inside this oracle.
 */
#include "dflash_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* storage widening                                                    */
/* ------------------------------------------------------------------ */

static inline double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static inline double wget(const void *w, int32_t dtype, size_t i) {
    return dtype == ORC_BF16 ? bf16_to_double(((const uint16_t *)w)[i])
                             : (double)((const float *)w)[i];
}

/* E4M3 (OCP 8-bit float, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities): sign * 2^(e-7) * (1 + m/8) for e > 0, sign * 2^-6 * (m/8) for
 * e = 0; codes 0x7F / 0xFF are NaN.  Written from that definition. */
double orc_e4m3_value(uint8_t c) {
    int32_t e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (c & 0x80) ? -mag : mag;
}

/* E2M1 (OCP 4-bit float: sign bit, 2 exponent bits with bias 1, 1 mantissa
 * bit, no infinities or NaN): sign * 2^(e-1) * (1 + m/2) for e > 0, sign * m/2
 * for e = 0.  Written from that definition. */
double orc_e2m1_value(uint8_t c) {
    int32_t e = (c >> 1) & 3, m = c & 1;
    double mag = e == 0 ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return (c & 8) ? -mag : mag;
}

/* Dot product of row `row` of an MXFP4 matrix: the quantised weight of element
 * k is scale[row] * 2^(E - 127) * e2m1_value(code_k), with E the block scale
 * byte of k's 32-value block (fp64), summed like the other dot products. */
static double dot_mxfp4(const orc_mxfp4 *q, size_t row, const double *x, int32_t K) {
    const uint8_t *c = q->codes + row * (size_t)(K / 2);
    const double sc = (double)q->scale[row];
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int32_t k = 0; k < K; ++k) {
        const uint8_t code = (k & 1) ? (uint8_t)(c[k / 2] >> 4) : (uint8_t)(c[k / 2] & 15);
        const uint8_t e = q->bscale[(((size_t)(k / 128) * (size_t)q->rows + row) * 4) + (size_t)((k / 32) % 4)];
        acc[k % 8] += sc * ldexp(orc_e2m1_value(code), (int)e - 127) * x[k];
    }
    return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

/* Dot product of one row of an FP8 matrix: the quantised weight of element k
 * is scale * e4m3_value(code_k) (fp64), summed like the other dot products. */
static double dot_fp8(const uint8_t *c, double scale, const double *x, int32_t K) {
    double a0 = 0, a1 = 0, a2 = 0, a3 = 0, a4 = 0, a5 = 0, a6 = 0, a7 = 0;
    int32_t k = 0;
    for (; k + 8 <= K; k += 8) {
        a0 += scale * orc_e4m3_value(c[k + 0]) * x[k + 0];
        a1 += scale * orc_e4m3_value(c[k + 1]) * x[k + 1];
        a2 += scale * orc_e4m3_value(c[k + 2]) * x[k + 2];
        a3 += scale * orc_e4m3_value(c[k + 3]) * x[k + 3];
        a4 += scale * orc_e4m3_value(c[k + 4]) * x[k + 4];
        a5 += scale * orc_e4m3_value(c[k + 5]) * x[k + 5];
        a6 += scale * orc_e4m3_value(c[k + 6]) * x[k + 6];
        a7 += scale * orc_e4m3_value(c[k + 7]) * x[k + 7];
    }
    double s = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
    for (; k < K; ++k) s += scale * orc_e4m3_value(c[k]) * x[k];
    return s;
}

static inline const void *wrow(const void *w, int32_t dtype, size_t elem_offset) {
    return dtype == ORC_BF16 ? (const void *)((const uint16_t *)w + elem_offset)
                             : (const void *)((const float *)w + elem_offset);
}

/* Dot products in 8 interleaved fp64 partial sums combined in a fixed order. */
static double dot_bf16(const uint16_t *w, const double *x, int32_t K) {
    double a0 = 0, a1 = 0, a2 = 0, a3 = 0, a4 = 0, a5 = 0, a6 = 0, a7 = 0;
    int32_t k = 0;
    for (; k + 8 <= K; k += 8) {
        a0 += bf16_to_double(w[k + 0]) * x[k + 0];
        a1 += bf16_to_double(w[k + 1]) * x[k + 1];
        a2 += bf16_to_double(w[k + 2]) * x[k + 2];
        a3 += bf16_to_double(w[k + 3]) * x[k + 3];
        a4 += bf16_to_double(w[k + 4]) * x[k + 4];
        a5 += bf16_to_double(w[k + 5]) * x[k + 5];
        a6 += bf16_to_double(w[k + 6]) * x[k + 6];
        a7 += bf16_to_double(w[k + 7]) * x[k + 7];
    }
    double s = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
    for (; k < K; ++k) s += bf16_to_double(w[k]) * x[k];
    return s;
}

static double dot_f32(const float *w, const double *x, int32_t K) {
    double a0 = 0, a1 = 0, a2 = 0, a3 = 0, a4 = 0, a5 = 0, a6 = 0, a7 = 0;
    int32_t k = 0;
    for (; k + 8 <= K; k += 8) {
        a0 += (double)w[k + 0] * x[k + 0];
        a1 += (double)w[k + 1] * x[k + 1];
        a2 += (double)w[k + 2] * x[k + 2];
        a3 += (double)w[k + 3] * x[k + 3];
        a4 += (double)w[k + 4] * x[k + 4];
        a5 += (double)w[k + 5] * x[k + 5];
        a6 += (double)w[k + 6] * x[k + 6];
        a7 += (double)w[k + 7] * x[k + 7];
    }
    double s = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
    for (; k < K; ++k) s += (double)w[k] * x[k];
    return s;
}

static double dot_f64(const double *a, const double *b, int32_t K) {
    double a0 = 0, a1 = 0, a2 = 0, a3 = 0, a4 = 0, a5 = 0, a6 = 0, a7 = 0;
    int32_t k = 0;
    for (; k + 8 <= K; k += 8) {
        a0 += a[k + 0] * b[k + 0];
        a1 += a[k + 1] * b[k + 1];
        a2 += a[k + 2] * b[k + 2];
        a3 += a[k + 3] * b[k + 3];
        a4 += a[k + 4] * b[k + 4];
        a5 += a[k + 5] * b[k + 5];
        a6 += a[k + 6] * b[k + 6];
        a7 += a[k + 7] * b[k + 7];
    }
    double s = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
    for (; k < K; ++k) s += a[k] * b[k];
    return s;
}

/* ------------------------------------------------------------------ */
/* building blocks                                                     */
/* ------------------------------------------------------------------ */

void orc_matmul_rows(const void *W, int32_t dtype, int32_t row0, int32_t N, int32_t K,
                     const double *X, int32_t R, double *Y) {
    /* Y[r][n] = sum_k W[row0 + n][k] * X[r][k]; each (r, n) is one dot_* call. */
#pragma omp parallel for schedule(static)
    for (int32_t n = 0; n < N; ++n) {
        const size_t row = (size_t)row0 + (size_t)n;
        for (int32_t r = 0; r < R; ++r) {
            double v;
            if (dtype == ORC_FP8) {
                const orc_fp8 *q = (const orc_fp8 *)W;
                v = dot_fp8(q->codes + row * K, (double)q->scale[row], X + (size_t)r * K, K);
            } else if (dtype == ORC_MXFP4) {
                v = dot_mxfp4((const orc_mxfp4 *)W, row, X + (size_t)r * K, K);
            } else if (dtype == ORC_BF16) {
                v = dot_bf16((const uint16_t *)W + row * K, X + (size_t)r * K, K);
            } else {
                v = dot_f32((const float *)W + row * K, X + (size_t)r * K, K);
            }
            Y[(size_t)r * N + n] = v;
        }
    }
}

void orc_matmul(const void *W, int32_t dtype, int32_t N, int32_t K,
                const double *X, int32_t R, double *Y) {
    orc_matmul_rows(W, dtype, 0, N, K, X, R, Y);
}

void orc_rmsnorm(const double *x, const float *g, int32_t n, double eps, double *y) {
    /* y = x / sqrt(mean(x^2) + eps) * g */
    double ss = 0.0;
    for (int32_t i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss / (double)n + eps);
    for (int32_t i = 0; i < n; ++i) y[i] = x[i] * inv * (double)g[i];
}

void orc_rope(double *v, int32_t hd, int64_t pos, double theta) {
    /* rotate pairs (i, i + hd/2) by angle pos * theta^(-2i/hd) */
    int32_t half = hd / 2;
    for (int32_t i = 0; i < half; ++i) {
        double freq = pow(theta, -2.0 * (double)i / (double)hd);
        double ang = (double)pos * freq;
        double c = cos(ang), s = sin(ang);
        double x1 = v[i], x2 = v[i + half];
        v[i] = x1 * c - x2 * s;
        v[i + half] = x2 * c + x1 * s;
    }
}

/* Fidelity toggle, not on the pages: the frequency rescaling published with
 * Llama 3.1 (its rope_scaling settings factor, low_freq_factor,
 * high_freq_factor, original_max_position_embeddings).  A pair whose
 * wavelength 2*pi/f is shorter than original_max / high_freq_factor keeps f;
 * one longer than original_max / low_freq_factor gets f / factor; in between
 * f / factor and f are mixed with weight
 * s = (original_max / wavelength - low_freq_factor) / (high_freq_factor - low_freq_factor)
 * on f, which is continuous at both band edges. */
double orc_rope_inv_freq(const orc_dims *d, int32_t i) {
    double f = pow(d->rope_theta, -2.0 * (double)i / (double)d->head_dim);
    if (!(d->rope_factor > 1.0)) return f;
    double wavelen = 2.0 * 3.14159265358979323846 / f;
    double lo_edge = d->rope_original_max_pos / d->rope_high_freq_factor;  /* shortest rescaled wavelength */
    double hi_edge = d->rope_original_max_pos / d->rope_low_freq_factor;   /* longest partly kept wavelength */
    if (wavelen < lo_edge) return f;
    if (wavelen > hi_edge) return f / d->rope_factor;
    double s = (d->rope_original_max_pos / wavelen - d->rope_low_freq_factor) /
               (d->rope_high_freq_factor - d->rope_low_freq_factor);
    return (1.0 - s) * f / d->rope_factor + s * f;
}

void orc_rope_dims(double *v, const orc_dims *d, int64_t pos) {
    int32_t hd = d->head_dim, half = hd / 2;
    if (!(d->rope_factor > 1.0)) {
        orc_rope(v, hd, pos, d->rope_theta);
        return;
    }
    for (int32_t i = 0; i < half; ++i) {
        double ang = (double)pos * orc_rope_inv_freq(d, i);
        double c = cos(ang), s = sin(ang);
        double x1 = v[i], x2 = v[i + half];
        v[i] = x1 * c - x2 * s;
        v[i + half] = x2 * c + x1 * s;
    }
}

/* Fidelity toggle, not on the pages: Qwen3 layers normalise every q and k head
 * (RMSNorm over head_dim with a per-dimension gain, the layer's rms_eps) before
 * RoPE.  In place on n_heads consecutive vectors of hd. */
static void qk_norm_heads(double *v, int32_t n_heads, int32_t hd, const float *g, double eps) {
    for (int32_t h = 0; h < n_heads; ++h) orc_rmsnorm(v + (size_t)h * hd, g, hd, eps, v + (size_t)h * hd);
}

void orc_attend(const double *q, const double *keys, const double *vals, int64_t ld_kv,
                int32_t n_keys, int32_t hd, double *out) {
    /* softmax_j(q . k_j / sqrt(hd)) weighted sum of v_j, keys in order 0..n-1 */
    double *s = (double *)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
    double scale = 1.0 / sqrt((double)hd);
    double mx = -INFINITY;
    for (int32_t j = 0; j < n_keys; ++j) {
        s[j] = dot_f64(q, keys + (size_t)j * ld_kv, hd) * scale;
        if (s[j] > mx) mx = s[j];
    }
    double den = 0.0;
    for (int32_t j = 0; j < n_keys; ++j) {
        s[j] = exp(s[j] - mx);
        den += s[j];
    }
    for (int32_t d = 0; d < hd; ++d) out[d] = 0.0;
    for (int32_t j = 0; j < n_keys; ++j) {
        const double *v = vals + (size_t)j * ld_kv;
        for (int32_t d = 0; d < hd; ++d) out[d] += s[j] * v[d];
    }
    if (n_keys > 0)
        for (int32_t d = 0; d < hd; ++d) out[d] /= den;
    free(s);
}

int32_t orc_argmax(const double *x, int32_t n, double *margin) {
    int32_t best = 0;
    for (int32_t i = 1; i < n; ++i)
        if (x[i] > x[best]) best = i;           /* strict: lowest index on ties */
    if (margin) {
        double second = -INFINITY;
        for (int32_t i = 0; i < n; ++i)
            if (i != best && x[i] > second) second = x[i];
        *margin = n > 1 ? x[best] - second : INFINITY;
    }
    return best;
}

int32_t orc_accept(const int32_t *drafts, const int32_t *g, int32_t B) {
    int32_t a = 0;
    while (a < B - 1 && drafts[a] == g[a]) ++a;   /* d_(a+1) == g_a */
    return a;
}

static inline double silu(double x) { return x / (1.0 + exp(-x)); }

static void swiglu_rows(const void *w_gate_up, const void *w_down, int32_t dtype,
                        int32_t H, int32_t F, const double *m, int32_t R, double *out) {
    double *gu = (double *)malloc(sizeof(double) * (size_t)R * 2 * F);
    double *h = (double *)malloc(sizeof(double) * (size_t)R * F);
    orc_matmul(w_gate_up, dtype, 2 * F, H, m, R, gu);
    for (int32_t r = 0; r < R; ++r)
        for (int32_t i = 0; i < F; ++i)
            h[(size_t)r * F + i] = silu(gu[(size_t)r * 2 * F + i]) * gu[(size_t)r * 2 * F + F + i];
    orc_matmul(w_down, dtype, H, F, h, R, out);
    free(gu);
    free(h);
}

static void moe_row(const orc_model *m, const orc_layer *L, const double *x, double *out) {
    const orc_dims *d = &m->d;
    int32_t E = d->n_experts, H = d->hidden, Fe = d->expert_ffn, K = d->top_k;
    double *r = (double *)malloc(sizeof(double) * (size_t)E);
    orc_matmul(L->w_router, m->mat_dtype, E, H, x, 1, r);
    double mx = -INFINITY;
    for (int32_t e = 0; e < E; ++e) if (r[e] > mx) mx = r[e];
    double den = 0.0;
    for (int32_t e = 0; e < E; ++e) { r[e] = exp(r[e] - mx); den += r[e]; }
    for (int32_t e = 0; e < E; ++e) r[e] /= den;
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    char *used = (char *)calloc((size_t)E, 1);
    double wsum = 0.0;
    for (int32_t k = 0; k < K; ++k) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e)
            if (!used[e] && (best < 0 || r[e] > r[best])) best = e;
        used[best] = 1;
        sel[k] = best;
        wsum += r[best];
    }
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    for (int32_t i = 0; i < H; ++i) out[i] = 0.0;
    for (int32_t k = 0; k < K; ++k) {
        int32_t e = sel[k];
        double w = r[e] / wsum;
        swiglu_rows(wrow(L->we_gate_up, m->mat_dtype, (size_t)e * 2 * Fe * H),
                    wrow(L->we_down, m->mat_dtype, (size_t)e * H * Fe), m->mat_dtype, H, Fe, x, 1, y);
        for (int32_t i = 0; i < H; ++i) out[i] += w * y[i];
    }
    free(y); free(used); free(sel); free(r);
}

void orc_ffn(const orc_model *m, int32_t layer, const double *x, double *out) {
    const orc_layer *L = &m->layers[layer];
    if (m->d.n_experts > 0) moe_row(m, L, x, out);
    else swiglu_rows(L->w_gate_up, L->w_down, m->mat_dtype, m->d.hidden, m->d.ffn, x, 1, out);
}

static void ffn_rows(const orc_model *m, int32_t layer, const double *xn, int32_t R, double *out) {
    const orc_layer *L = &m->layers[layer];
    int32_t H = m->d.hidden;
    if (m->d.n_experts > 0) {
#pragma omp parallel for schedule(dynamic, 1) if (R > 1)
        for (int32_t r = 0; r < R; ++r) moe_row(m, L, xn + (size_t)r * H, out + (size_t)r * H);
    } else {
        swiglu_rows(L->w_gate_up, L->w_down, m->mat_dtype, H, m->d.ffn, xn, R, out);
    }
}

void orc_fuse(const orc_spec *s, const double *taps, double *c) {
    int32_t H = s->target.d.hidden, Hd = s->drafter.d.hidden;
    double *u = (double *)malloc(sizeof(double) * (size_t)Hd);
    orc_matmul(s->w_fc, s->drafter.mat_dtype, Hd, s->n_taps * H, taps, 1, u);
    orc_rmsnorm(u, s->fc_norm, Hd, s->drafter.d.rms_eps, c);
    free(u);
}

/* ------------------------------------------------------------------ */
/* sessions                                                            */
/* ------------------------------------------------------------------ */

struct orc_session {
    orc_spec s;
    int32_t max_len;
    int32_t len;        /* valid target KV positions = position of the anchor */
    int32_t ctx_len;    /* valid drafter context positions */
    double *tk, *tv;    /* target KV [Lt][max_len][nkv*hd] */
    double *dk, *dv;    /* drafter KV [Ld][max_len][nkv*hd]; context then scratch */
    double *taps;       /* [rows][n_taps][H] of the last target pass */
    int32_t taps_cap, taps_rows, taps_pos0;
};

static size_t kvw(const orc_dims *d) { return (size_t)d->n_kv_heads * d->head_dim; }

orc_session *orc_session_new(const orc_spec *s, int32_t max_len) {
    orc_session *ss = (orc_session *)calloc(1, sizeof *ss);
    ss->s = *s;
    ss->max_len = max_len;
    size_t nt = (size_t)s->target.d.n_layers * max_len * kvw(&s->target.d);
    size_t nd = (size_t)s->drafter.d.n_layers * max_len * kvw(&s->drafter.d);
    ss->tk = (double *)calloc(nt ? nt : 1, sizeof(double));
    ss->tv = (double *)calloc(nt ? nt : 1, sizeof(double));
    ss->dk = (double *)calloc(nd ? nd : 1, sizeof(double));
    ss->dv = (double *)calloc(nd ? nd : 1, sizeof(double));
    return ss;
}

void orc_session_free(orc_session *ss) {
    if (!ss) return;
    free(ss->tk); free(ss->tv); free(ss->dk); free(ss->dv); free(ss->taps);
    free(ss);
}

int32_t orc_session_len(const orc_session *ss) { return ss->len; }
const double *orc_last_taps(const orc_session *ss) { return ss->taps; }

static double *tkv_at(double *base, const orc_dims *d, int32_t max_len, int32_t l, int32_t t) {
    return base + ((size_t)l * max_len + t) * kvw(d);
}

void orc_ctx_kv(const orc_session *ss, int32_t j, int32_t t, double *k, double *v) {
    const orc_dims *d = &ss->s.drafter.d;
    memcpy(k, tkv_at(ss->dk, d, ss->max_len, j, t), sizeof(double) * kvw(d));
    memcpy(v, tkv_at(ss->dv, d, ss->max_len, j, t), sizeof(double) * kvw(d));
}

void orc_target_kv(const orc_session *ss, int32_t l, int32_t t, double *k, double *v) {
    const orc_dims *d = &ss->s.target.d;
    memcpy(k, tkv_at(ss->tk, d, ss->max_len, l, t), sizeof(double) * kvw(d));
    memcpy(v, tkv_at(ss->tv, d, ss->max_len, l, t), sizeof(double) * kvw(d));
}

static void embed_rows(const orc_model *emb_owner, const int32_t *tokens, int32_t R, double *x) {
    int32_t H = emb_owner->d.hidden;
    for (int32_t r = 0; r < R; ++r)
        for (int32_t i = 0; i < H; ++i)
            x[(size_t)r * H + i] = wget(emb_owner->embed, emb_owner->dtype, (size_t)tokens[r] * H + i);
}

/* Attention sub-block of one decoder layer over R rows whose keys/values are
 * already in the layer's cache.  Row r sees cache positions [0, n_keys(r)). */
static void attn_rows(const orc_dims *d, const double *q, const double *kc, const double *vc,
                      const int32_t *n_keys, int32_t R, double *att) {
    int32_t hd = d->head_dim, nq = d->n_q_heads, nkv = d->n_kv_heads, grp = nq / nkv;
    int64_t ld = (int64_t)nkv * hd;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t r = 0; r < R; ++r)
        for (int32_t h = 0; h < nq; ++h) {
            int32_t g = h / grp;
            orc_attend(q + ((size_t)r * nq + h) * hd, kc + (size_t)g * hd, vc + (size_t)g * hd, ld,
                       n_keys[r], hd, att + ((size_t)r * nq + h) * hd);
        }
}

/* One decoder layer (R1) on rows x[R][H] at positions pos0..pos0+R-1.
 * K/V of the rows are written to kc/vc (layer slabs of max_len positions);
 * row r attends over [0, n_keys[r]). */
static void layer_rows(const orc_model *m, int32_t l, double *x, int32_t R, int32_t pos0,
                       double *kc, double *vc, const int32_t *n_keys) {
    const orc_dims *d = &m->d;
    const orc_layer *L = &m->layers[l];
    int32_t H = d->hidden, hd = d->head_dim, nq = d->n_q_heads, nkv = d->n_kv_heads;
    int32_t qd = nq * hd, kd = nkv * hd, nqkv = qd + 2 * kd;
    double *n = (double *)calloc((size_t)R * H, sizeof(double));
    double *qkv = (double *)malloc(sizeof(double) * (size_t)R * nqkv);
    double *q = (double *)malloc(sizeof(double) * (size_t)R * qd);
    double *att = (double *)malloc(sizeof(double) * (size_t)R * qd);
    double *o = (double *)malloc(sizeof(double) * (size_t)R * H);
    for (int32_t r = 0; r < R; ++r) orc_rmsnorm(x + (size_t)r * H, L->attn_norm, H, d->rms_eps, n + (size_t)r * H);
    orc_matmul(L->wqkv, m->mat_dtype, nqkv, H, n, R, qkv);
    for (int32_t r = 0; r < R; ++r) {
        const double *row = qkv + (size_t)r * nqkv;
        int32_t pos = pos0 + r;
        memcpy(q + (size_t)r * qd, row, sizeof(double) * qd);
        if (d->qk_norm) qk_norm_heads(q + (size_t)r * qd, nq, hd, L->q_norm, d->rms_eps);
        for (int32_t h = 0; h < nq; ++h) orc_rope_dims(q + (size_t)r * qd + (size_t)h * hd, d, pos);
        double *kp = kc + (size_t)pos * kd, *vp = vc + (size_t)pos * kd;
        memcpy(kp, row + qd, sizeof(double) * kd);
        memcpy(vp, row + qd + kd, sizeof(double) * kd);
        if (d->qk_norm) qk_norm_heads(kp, nkv, hd, L->k_norm, d->rms_eps);
        for (int32_t g = 0; g < nkv; ++g) orc_rope_dims(kp + (size_t)g * hd, d, pos);
    }
    attn_rows(d, q, kc, vc, n_keys, R, att);
    orc_matmul(L->wo, m->mat_dtype, H, qd, att, R, o);
    for (size_t i = 0; i < (size_t)R * H; ++i) x[i] += o[i];
    for (int32_t r = 0; r < R; ++r) orc_rmsnorm(x + (size_t)r * H, L->ffn_norm, H, d->rms_eps, n + (size_t)r * H);
    ffn_rows(m, l, n, R, o);
    for (size_t i = 0; i < (size_t)R * H; ++i) x[i] += o[i];
    free(n); free(qkv); free(q); free(att); free(o);
}

static void head_rows(const orc_model *m, const void *lm_head, int32_t lm_dtype, int32_t V,
                      const double *x, int32_t R, double *logits) {
    int32_t H = m->d.hidden;
    double *xn = (double *)malloc(sizeof(double) * (size_t)R * H);
    for (int32_t r = 0; r < R; ++r) orc_rmsnorm(x + (size_t)r * H, m->final_norm, H, m->d.rms_eps, xn + (size_t)r * H);
    orc_matmul(lm_head, lm_dtype, V, H, xn, R, logits);
    free(xn);
}

/* Target forward (causal) on R rows at positions len..len+R-1; stores taps;
 * returns the final residual rows in x. */
static void target_rows(orc_session *ss, const int32_t *tokens, int32_t R, double *x) {
    const orc_model *m = &ss->s.target;
    const orc_dims *d = &m->d;
    int32_t H = d->hidden, nt = ss->s.n_taps, p0 = ss->len;
    if (ss->taps_cap < R) {
        free(ss->taps);
        ss->taps = (double *)malloc(sizeof(double) * (size_t)R * nt * H);
        ss->taps_cap = R;
    }
    int32_t *nk = (int32_t *)malloc(sizeof(int32_t) * (size_t)R);
    for (int32_t r = 0; r < R; ++r) nk[r] = p0 + r + 1;   /* causal */
    embed_rows(m, tokens, R, x);
    for (int32_t l = 0; l < d->n_layers; ++l) {
        layer_rows(m, l, x, R, p0, tkv_at(ss->tk, d, ss->max_len, l, 0),
                   tkv_at(ss->tv, d, ss->max_len, l, 0), nk);
        for (int32_t t = 0; t < nt; ++t)
            if (ss->s.tap_layers[t] == l)
                for (int32_t r = 0; r < R; ++r)
                    memcpy(ss->taps + ((size_t)r * nt + t) * H, x + (size_t)r * H, sizeof(double) * H);
    }
    ss->taps_rows = R;
    ss->taps_pos0 = p0;
    free(nk);
}

/* Context K/V injection (R4, R5) for tap rows 0..n-1 at positions pos0.. */
static void inject_ctx(orc_session *ss, int32_t n_rows, int32_t pos0) {
    const orc_model *m = &ss->s.drafter;
    const orc_dims *d = &m->d;
    int32_t Ht = ss->s.target.d.hidden, Hd = d->hidden, nt = ss->s.n_taps;
    int32_t hd = d->head_dim, qd = d->n_q_heads * hd, kd = d->n_kv_heads * hd;
    double *c = (double *)malloc(sizeof(double) * (size_t)n_rows * Hd);
    double *kv = (double *)malloc(sizeof(double) * (size_t)n_rows * 2 * kd);
    for (int32_t r = 0; r < n_rows; ++r) orc_fuse(&ss->s, ss->taps + (size_t)r * nt * Ht, c + (size_t)r * Hd);
    for (int32_t j = 0; j < d->n_layers; ++j) {
        /* rows qd..qd+2kd of Wqkv_j are [Wk_j; Wv_j] */
        orc_matmul_rows(m->layers[j].wqkv, m->mat_dtype, qd, 2 * kd, Hd, c, n_rows, kv);
        for (int32_t r = 0; r < n_rows; ++r) {
            int32_t t = pos0 + r;
            double *kp = tkv_at(ss->dk, d, ss->max_len, j, t), *vp = tkv_at(ss->dv, d, ss->max_len, j, t);
            memcpy(kp, kv + (size_t)r * 2 * kd, sizeof(double) * kd);
            memcpy(vp, kv + (size_t)r * 2 * kd + kd, sizeof(double) * kd);
            /* the context keys pass the same k processing as the block's keys (R5) */
            if (d->qk_norm) qk_norm_heads(kp, d->n_kv_heads, hd, m->layers[j].k_norm, d->rms_eps);
            for (int32_t g = 0; g < d->n_kv_heads; ++g) orc_rope_dims(kp + (size_t)g * hd, d, t);
        }
    }
    free(c); free(kv);
}

static int32_t prefill_impl(orc_session *ss, const int32_t *prompt, int32_t n, double *last_logits,
                            double *margin, int with_ctx) {
    const orc_model *m = &ss->s.target;
    int32_t H = m->d.hidden, V = m->d.vocab;
    double *x = (double *)malloc(sizeof(double) * (size_t)n * H);
    double *lg = (double *)malloc(sizeof(double) * (size_t)V);
    ss->len = 0;
    target_rows(ss, prompt, n, x);
    head_rows(m, m->lm_head, m->mat_dtype, V, x + (size_t)(n - 1) * H, 1, lg);
    int32_t tok = orc_argmax(lg, V, margin);
    if (last_logits) memcpy(last_logits, lg, sizeof(double) * V);
    if (with_ctx) inject_ctx(ss, n, 0);
    ss->len = n;
    ss->ctx_len = with_ctx ? n : 0;
    free(x); free(lg);
    return tok;
}

int32_t orc_prefill(orc_session *ss, const int32_t *prompt, int32_t n, double *last_logits, double *margin) {
    return prefill_impl(ss, prompt, n, last_logits, margin, 1);
}

void orc_draft(orc_session *ss, int32_t anchor, int32_t *drafts, double *logits, double *margins) {
    const orc_model *m = &ss->s.drafter, *t = &ss->s.target;
    const orc_dims *d = &m->d;
    int32_t B = ss->s.block_size, H = d->hidden, V = t->d.vocab, p = ss->ctx_len;
    int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    int32_t *nk = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    double *x = (double *)malloc(sizeof(double) * (size_t)B * H);
    double *lg = (double *)malloc(sizeof(double) * (size_t)(B > 1 ? B - 1 : 1) * V);
    tok[0] = anchor;
    for (int32_t r = 1; r < B; ++r) tok[r] = ss->s.mask_token_id;
    for (int32_t r = 0; r < B; ++r) nk[r] = p + B;         /* block-bidirectional */
    embed_rows(t, tok, B, x);                               /* target's table (R6) */
    for (int32_t j = 0; j < d->n_layers; ++j)
        layer_rows(m, j, x, B, p, tkv_at(ss->dk, d, ss->max_len, j, 0),
                   tkv_at(ss->dv, d, ss->max_len, j, 0), nk);
    if (B > 1) {
        head_rows(m, t->lm_head, t->mat_dtype, V, x + H, B - 1, lg);
        for (int32_t r = 0; r < B - 1; ++r)
            drafts[r] = orc_argmax(lg + (size_t)r * V, V, margins ? margins + r : NULL);
        if (logits) memcpy(logits, lg, sizeof(double) * (size_t)(B - 1) * V);
    }
    free(tok); free(nk); free(x); free(lg);
}

void orc_verify(orc_session *ss, const int32_t *tokens, int32_t *g, double *logits, double *margins) {
    const orc_model *m = &ss->s.target;
    int32_t B = ss->s.block_size, H = m->d.hidden, V = m->d.vocab;
    double *x = (double *)malloc(sizeof(double) * (size_t)B * H);
    double *lg = (double *)malloc(sizeof(double) * (size_t)B * V);
    target_rows(ss, tokens, B, x);
    head_rows(m, m->lm_head, m->mat_dtype, V, x, B, lg);
    for (int32_t r = 0; r < B; ++r) g[r] = orc_argmax(lg + (size_t)r * V, V, margins ? margins + r : NULL);
    if (logits) memcpy(logits, lg, sizeof(double) * (size_t)B * V);
    free(x); free(lg);
}

int32_t orc_commit(orc_session *ss, int32_t a) {
    inject_ctx(ss, a + 1, ss->len);
    ss->len += a + 1;
    ss->ctx_len = ss->len;
    return ss->len;
}

/* ------------------------------------------------------------------ */
/* whole generations                                                   */
/* ------------------------------------------------------------------ */

void orc_generate_ar(const orc_spec *s, const int32_t *prompt, int32_t n, int32_t max_new,
                     int32_t *out, double *margins) {
    orc_session *ss = orc_session_new(s, n + max_new + 1);
    const orc_model *m = &s->target;
    int32_t H = m->d.hidden, V = m->d.vocab;
    double *x = (double *)malloc(sizeof(double) * (size_t)H);
    double *lg = (double *)malloc(sizeof(double) * (size_t)V);
    if (max_new > 0) out[0] = prefill_impl(ss, prompt, n, NULL, margins ? margins : NULL, 0);
    for (int32_t i = 1; i < max_new; ++i) {
        target_rows(ss, out + i - 1, 1, x);
        ss->len += 1;
        head_rows(m, m->lm_head, m->mat_dtype, V, x, 1, lg);
        out[i] = orc_argmax(lg, V, margins ? margins + i : NULL);
    }
    free(x); free(lg);
    orc_session_free(ss);
}

int32_t orc_generate_spec(const orc_spec *s, const int32_t *prompt, int32_t n, int32_t max_new,
                          const int32_t *forced, int32_t *out, int32_t *accept_log) {
    int32_t B = s->block_size;
    orc_session *ss = orc_session_new(s, n + max_new + 2 * B);
    int32_t *drafts = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    int32_t *blk = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    int32_t *g = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    int32_t it = 0, n_out = 0;
    if (max_new <= 0) goto done;
    int32_t anchor = orc_prefill(ss, prompt, n, NULL, NULL);
    out[n_out++] = anchor;
    while (n_out < max_new) {
        if (forced) for (int32_t i = 0; i < B - 1; ++i) drafts[i] = forced[n_out + i];
        else orc_draft(ss, anchor, drafts, NULL, NULL);
        blk[0] = anchor;
        for (int32_t i = 1; i < B; ++i) blk[i] = drafts[i - 1];
        orc_verify(ss, blk, g, NULL, NULL);
        int32_t a = orc_accept(drafts, g, B);
        orc_commit(ss, a);
        for (int32_t i = 0; i < a && n_out < max_new; ++i) out[n_out++] = drafts[i];
        if (n_out < max_new) out[n_out++] = g[a];
        anchor = g[a];
        if (accept_log) accept_log[it] = a;
        ++it;
    }
done:
    free(drafts); free(blk); free(g);
    orc_session_free(ss);
    return it;
}
