/*
 * dflash_oracle.h -- plain, slow fp64 CPU oracle of the DFlash draft-and-verify
 * decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product library
 * never includes, links or calls anything here, and nothing here uses the
 * product's code.
 *
 * Sources (web pages about DFlash, cited by title and section):
 *  [P1] forbuilders.ai, "Nova técnica faz modelo Qwen rodar a mais de 1.000
 *       tokens por segundo", section "Como funciona a decodificação especulativa".
 *  [P2] iaemfoco.com, "DFlash: Decodificação Especulativa com Blocos em Paralelo
 *       Alcança Até 15x Mais Throughput em GPUs Blackwell", sections
 *       "Decodificação especulativa tradicional", "O que o DFlash faz de
 *       diferente", "O alvo sabe mais", "Drafter leve, ganho máximo", "Como usar".
 *  [P4] imasters.com.br, "NVIDIA acelera LLMs autorregressivos em até 15 vezes",
 *       sections "Como o DFlash troca o drafter por difusão de blocos" and
 *       "Os três mecanismos por trás do DFlash".
 *  [P5] ceviu.com.br, "DFlash e Spec V2 revolucionam a speculative decoding".
 *
 * Everything the pages leave open follows one stated reading (see the .c file).
 * All arithmetic is IEEE fp64.  Matrix weights are read from fp32 or bf16
 * storage and widened exactly to fp64, or from FP8 codes with per-row scales
 * (scale * E4M3 value, in fp64).
 */
#ifndef DFLASH_ORACLE_H
#define DFLASH_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8 = 2, ORC_MXFP4 = 3 };

/* A matrix in FP8 storage: E4M3 codes [rows][K] and one fp32 scale per row;
 * the quantised weight is scale[row] * e4m3_value(code).  Matrix pointers of
 * an ORC_FP8 model point to one of these. */
typedef struct {
    const uint8_t *codes;
    const float *scale;
} orc_fp8;

/* A matrix in MXFP4 storage (OCP Microscaling: FP4 E2M1 elements sharing a
 * power-of-two scale per 32 values along K) with one fp32 scale per row:
 * codes [rows][K/2] (element k in byte k/2, low nibble for even k), bscale
 * [K/128][rows][4] (byte (k/128, row, (k/32) % 4) = the block's exponent + 127),
 * scale [rows].  The quantised weight of element (row, k) is
 * scale[row] * 2^(bscale byte - 127) * e2m1_value(code).  Matrix pointers of an
 * ORC_MXFP4 model point to one of these. */
typedef struct {
    const uint8_t *codes;
    const uint8_t *bscale;
    const float *scale;
    int64_t rows;             /* rows of the whole matrix (the bscale row stride) */
} orc_mxfp4;

typedef struct {
    int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    int32_t n_experts, top_k, expert_ffn;   /* n_experts == 0: dense SwiGLU */
    double rms_eps, rope_theta;
    /* fidelity toggles, off by default (not on the pages):
     * qk_norm: per-head RMSNorm of q and k before RoPE (Qwen3 layers);
     * rope_factor > 1: Llama 3.1 rescaling of the RoPE frequencies. */
    int32_t qk_norm;
    double rope_factor, rope_low_freq_factor, rope_high_freq_factor, rope_original_max_pos;
} orc_dims;

typedef struct {
    const float *attn_norm;   /* [H] */
    const void *wqkv;         /* [(nq+2nkv)*hd, H], rows [Wq; Wk; Wv] */
    const void *wo;           /* [H, nq*hd] */
    const float *ffn_norm;    /* [H] */
    const void *w_gate_up;    /* dense: [2F, H], rows [W_gate; W_up] */
    const void *w_down;       /* dense: [H, F] */
    const void *w_router;     /* MoE: [E, H] */
    const void *we_gate_up;   /* MoE: [E, 2Fe, H] */
    const void *we_down;      /* MoE: [E, H, Fe] */
    const float *q_norm;      /* qk_norm: [hd] gain of every q head */
    const float *k_norm;      /* qk_norm: [hd] gain of every k head */
} orc_layer;

typedef struct {
    orc_dims d;
    int32_t dtype;            /* storage type of the embedding: ORC_F32 / ORC_BF16 */
    const void *embed;        /* [V, H] (the drafter uses the target's) */
    const void *lm_head;      /* [V, H] (the drafter uses the target's) */
    const float *final_norm;  /* [H] */
    const orc_layer *layers;  /* [n_layers] */
    int32_t mat_dtype;        /* storage of the projection matrices, the LM head and W_fc:
                                 ORC_F32, ORC_BF16, ORC_FP8 (pointers to orc_fp8) or
                                 ORC_MXFP4 (pointers to orc_mxfp4) */
} orc_model;

typedef struct {
    orc_model target, drafter;
    int32_t block_size;       /* B: anchor + (B-1) mask positions */
    int32_t n_taps;
    const int32_t *tap_layers;
    int32_t mask_token_id;
    const void *w_fc;         /* [H, n_taps*H] */
    const float *fc_norm;     /* [H] */
} orc_spec;

typedef struct orc_session orc_session;

/* ---- building blocks (each pinned separately by the tests) ---- */
void orc_rmsnorm(const double *x, const float *g, int32_t n, double eps, double *y);
void orc_rope(double *v, int32_t head_dim, int64_t pos, double theta);
/* Inverse frequency of RoPE pair i under the model's settings (theta^(-2i/hd),
 * rescaled when rope_factor > 1), and the rotation with those frequencies. */
double orc_rope_inv_freq(const orc_dims *d, int32_t i);
void orc_rope_dims(double *v, const orc_dims *d, int64_t pos);
/* Y[r][n] = sum_k W[n][k] X[r][k]; W in fp32 / bf16 / FP8 storage. */
void orc_matmul(const void *W, int32_t dtype, int32_t N, int32_t K,
                const double *X, int32_t R, double *Y);
/* The same over rows row0 .. row0+N-1 of W. */
void orc_matmul_rows(const void *W, int32_t dtype, int32_t row0, int32_t N, int32_t K,
                     const double *X, int32_t R, double *Y);
/* Value of an E4M3 code (NaN for 0x7F / 0xFF). */
double orc_e4m3_value(uint8_t code);
/* Value of a 4-bit E2M1 code (0..15). */
double orc_e2m1_value(uint8_t code);
/* One query row over keys[0..n_keys) (each hd doubles, stride ld_k); softmax scale 1/sqrt(hd). */
void orc_attend(const double *q, const double *keys, const double *vals, int64_t ld_kv,
                int32_t n_keys, int32_t head_dim, double *out);
/* Index of the largest value (lowest index on exact ties) and top1 - top2 margin. */
int32_t orc_argmax(const double *x, int32_t n, double *margin);
/* a = largest k <= B-1 with drafts[i-1] == g[i-1] for all 1 <= i <= k (drafts are d_1..d_{B-1}). */
int32_t orc_accept(const int32_t *drafts, const int32_t *g, int32_t block_size);
/* Dense or MoE SwiGLU FFN of one layer on one normalised row m -> out[H]. */
void orc_ffn(const orc_model *m, int32_t layer, const double *x_normed, double *out);
/* Context vector c = RMSNorm(W_fc . concat(taps)); taps: [n_taps][H]. */
void orc_fuse(const orc_spec *s, const double *taps, double *c);

/* ---- sessions: one sequence of target + drafter state ---- */
orc_session *orc_session_new(const orc_spec *s, int32_t max_len);
void orc_session_free(orc_session *ss);
int32_t orc_session_len(const orc_session *ss);
/* Target over the prompt; writes target KV, fuses taps into drafter context
 * K/V for all prompt positions.  Returns the first greedy token (the anchor).
 * last_logits: [V] or NULL; margin: top1-top2 at the last row or NULL. */
int32_t orc_prefill(orc_session *ss, const int32_t *prompt, int32_t n,
                    double *last_logits, double *margin);
/* One drafter forward on [anchor, mask x (B-1)] at positions p..p+B-1.
 * drafts: [B-1]; logits: [(B-1)*V] or NULL; margins: [B-1] or NULL. */
void orc_draft(orc_session *ss, int32_t anchor, int32_t *drafts, double *logits, double *margins);
/* Target forward on tokens[0..B) at positions p..p+B-1, causal; KV written tentatively.
 * g: [B] greedy argmax per row; logits [B*V] or NULL; margins [B] or NULL. */
void orc_verify(orc_session *ss, const int32_t *tokens, int32_t *g, double *logits, double *margins);
/* Commit verify rows 0..a: target length p <- p+a+1, drafter context gets
 * positions p..p+a from the taps of those rows.  Returns the new length. */
int32_t orc_commit(orc_session *ss, int32_t a);
/* Hidden state h^(l) of the last verify (or prefill) rows, for inspection. */
const double *orc_last_taps(const orc_session *ss);
/* Drafter context K/V of layer j at position t (hd * n_kv doubles each). */
void orc_ctx_kv(const orc_session *ss, int32_t j, int32_t t, double *k_out, double *v_out);
/* Target KV of layer l at position t. */
void orc_target_kv(const orc_session *ss, int32_t l, int32_t t, double *k_out, double *v_out);

/* ---- whole generations ---- */
/* Target-only greedy decoding: out[0..max_new) after the prompt.
 * margins: [max_new] (top1-top2 of the logits each token was taken from) or NULL. */
void orc_generate_ar(const orc_spec *s, const int32_t *prompt, int32_t n, int32_t max_new,
                     int32_t *out, double *margins);
/* Draft-and-verify greedy decoding.  forced: NULL (use the drafter) or a
 * token script; when given, drafts d_1..d_{B-1} of each iteration are taken
 * from forced[n_out .. n_out+B-2] (the tokens a perfect drafter would propose
 * when forced holds the target-only continuation).
 * accept_log: one a per iteration (capacity max_new); returns iterations. */
int32_t orc_generate_spec(const orc_spec *s, const int32_t *prompt, int32_t n, int32_t max_new,
                          const int32_t *forced, int32_t *out, int32_t *accept_log);

#ifdef __cplusplus
}
#endif
#endif
