/*
 * dflash.h -- C ABI of the DFlash block-diffusion draft-and-verify decode
 * library for NVIDIA B200 (sm_100a).
 *
 * The method (web pages about DFlash, cited by title and section):
 *  - "DFlash: Decodificação Especulativa com Blocos em Paralelo Alcança Até 15x
 *    Mais Throughput em GPUs Blackwell" (iaemfoco.com), sections "O que o DFlash
 *    faz de diferente" (a light block-diffusion drafter proposes a whole block
 *    in one forward pass; the target verifies the whole block in parallel),
 *    "O alvo sabe mais" (hidden states of several target layers are fused into
 *    a compact context vector injected into the Key and Value projections of
 *    every drafter layer, where it persists in the KV cache),
 *    "Decodificação especulativa tradicional" (accepted tokens are kept; output
 *    identical to target-only decoding) and "Como usar" (15 speculative tokens).
 *  - "NVIDIA acelera LLMs autorregressivos em até 15 vezes" (imasters.com.br),
 *    sections "Como o DFlash troca o drafter por difusão de blocos" and "Os três
 *    mecanismos por trás do DFlash".
 *  - "DFlash e Spec V2 revolucionam a speculative decoding" (ceviu.com.br): 16
 *    tokens per drafter pass, K/V injection into every drafter layer, minimal
 *    host-device synchronisation.
 *
 * Conventions for every entry point:
 *  - Status codes are returned; no exception crosses the ABI.  Out-parameters
 *    are written only when DFLASH_OK is returned.  After DFLASH_ECUDA the
 *    context is unusable and must be destroyed.
 *  - Host pointers (const int32_t *prompt, int32_t *drafts ...) are ordinary
 *    host memory owned by the caller.  Calls that return results through host
 *    pointers synchronise the context's stream, bounded by a host-side timeout
 *    (DFLASH_ETIMEOUT).
 *  - Device memory: the caller allocates two device arenas (weights, state) of
 *    the sizes dflash_workspace_size reports and keeps them alive until
 *    dflash_destroy.  The library allocates no device memory of its own.
 *  - All GPU work is enqueued on the CUDA stream given to dflash_create, on
 *    the device that was current at dflash_create; every call makes that
 *    device current for its duration and restores the caller's afterwards.
 *  - A context is not thread-safe; use one context per host thread.
 */
#ifndef DFLASH_H
#define DFLASH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dflash_ctx dflash_ctx;

typedef enum {
    DFLASH_OK = 0,
    DFLASH_EINVAL = 1,     /* bad argument (null pointer, size out of range, unknown name) */
    DFLASH_ESTATE = 2,     /* call out of order (verify without draft, sequence not prefilled) */
    DFLASH_ECAPACITY = 3,  /* a sequence would exceed max_len / a batch exceeds max_batch */
    DFLASH_ECUDA = 4,      /* a CUDA call failed; the context must be destroyed */
    DFLASH_ENUMERIC = 5,   /* a non-finite value reached an argmax (device status word) */
    DFLASH_ETIMEOUT = 6,   /* the stream did not finish within the host-side timeout */
    DFLASH_EUNSUPPORTED = 7/* shape the kernels do not support (e.g. head_dim not 64/128) */
} dflash_status;

/* Model dtypes.  FP32: fp32 weights and activations.  BF16: bf16 weights;
 * activations (GEMM inputs, q, the K/V caches) carried as two bf16 planes,
 * hi = bf16(v) and lo = bf16(v - hi), so each bf16 tensor-core product takes
 * two (attention: three) MMAs and the result keeps ~16 significant bits --
 * weight bytes are unchanged, activation and K/V bytes double.  BF16_FAST:
 * bf16 weights and single-plane bf16 activations (half the K/V bytes and MMAs,
 * with the rounding error of plain bf16 inference).  FP8: every projection
 * matrix (Wqkv, Wo, gate/up, down, the LM head, the fuse W_fc) stored as E4M3
 * codes (1 byte; OCP 8-bit float, exponent bias 7, no infinities) with one fp32
 * scale per output row in the slot "<name>.scale", the embedding in bf16,
 * activations as for BF16; the model computed is the quantised one,
 * W[r][k] = scale[r] * e4m3_value(code[r][k]), so the greedy output equals the
 * quantised target's own greedy decoding.  Weight bytes per step halve.
 * FP4: the same matrices in MXFP4 (OCP Microscaling): 4-bit E2M1 codes, two per
 * byte (element k of a row in byte k/2, the low nibble for even k; 1 sign, 2
 * exponent bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6), one power-of-two exponent per 32 values of a row in "<name>.bscale"
 * [K/128][rows][4] (byte (k/128, r, (k/32) % 4) = exponent + 127, UE8M0) and
 * one fp32 scale per row in "<name>.scale"; W[r][k] = scale[r] *
 * 2^(bscale - 127) * e2m1_value(code[r][k]).  Weight bytes per step ~quarter.
 * Every K (hidden, ffn, q width, n_taps * hidden) a multiple of 128.
 * FP8 and FP4: dense models only (MoE targets: EINVAL). */
enum { DFLASH_FP32 = 0, DFLASH_BF16 = 1, DFLASH_BF16_FAST = 2, DFLASH_FP8 = 3, DFLASH_FP4 = 4 };
/* Storage type of the "<name>.bscale" weight slots (dflash_weight_info): bytes. */
enum { DFLASH_UE8M0 = 5 };

/* Draft modes.  MODEL: drafts are the drafter's argmax.  SCRIPT: the drafter
 * still runs in full, then its drafts are replaced from a per-sequence token
 * script (dflash_set_script): drafts d_1..d_{tau-1} are taken from the script
 * and d_tau is made wrong ((script+1) mod vocab), so each iteration commits
 * exactly tau tokens when the script is the target's own greedy continuation.
 * tau = block_size makes every draft come from the script. */
enum { DFLASH_DRAFT_MODEL = 0, DFLASH_DRAFT_SCRIPT = 1 };

#define DFLASH_MAX_TAPS 8
#define DFLASH_MAX_BLOCK 32

typedef struct {
    int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    int32_t n_experts, top_k, expert_ffn;   /* n_experts == 0: dense SwiGLU FFN */
    double rms_eps, rope_theta;
    /* Fidelity toggles of real checkpoints (not on the DFlash pages; 0 = off).
     * qk_norm = 1: every q and k head is RMS-normalised over head_dim (gain
     * slots q_norm / k_norm [head_dim] per layer, eps rms_eps) before RoPE, as
     * in Qwen3 layers; the drafter's context keys too.  rope_factor > 1: the
     * RoPE frequencies are rescaled as published with Llama 3.1 -- a pair whose
     * wavelength 2*pi/f is below rope_original_max_pos / rope_high_freq_factor
     * keeps f, one above rope_original_max_pos / rope_low_freq_factor gets
     * f / rope_factor, and in between the two are mixed with weight
     * (rope_original_max_pos / wavelength - low) / (high - low) on f. */
    int32_t qk_norm;
    int32_t reserved;             /* 0 */
    double rope_factor, rope_low_freq_factor, rope_high_freq_factor, rope_original_max_pos;
} dflash_model_cfg;

typedef struct {
    dflash_model_cfg target;      /* the model whose greedy output is reproduced */
    dflash_model_cfg drafter;     /* dense; drafter.vocab == target.vocab, same hidden */
    int32_t block_size;           /* B in [1, 32]: anchor + (B-1) drafted tokens */
    int32_t n_taps;               /* target layers whose outputs feed the context vector */
    int32_t tap_layers[DFLASH_MAX_TAPS];
    int32_t mask_token_id;        /* id embedded at block positions 1..B-1 */
    int32_t max_batch;            /* sequences held at once */
    int32_t max_len;              /* positions per sequence (prompt + generated + B) */
    int32_t prefill_chunk;        /* prompt rows per prefill pass (0: default 1024) */
    int32_t dtype;                /* DFLASH_FP32, DFLASH_BF16, DFLASH_BF16_FAST, DFLASH_FP8 or DFLASH_FP4 (see above) */
    int32_t keep_logits;          /* 1: keep fp32 logits of the last draft/verify for dflash_debug_logits */
    int32_t timeout_ms;           /* host wait bound for synchronising calls (0: 600000) */
    int32_t sampling;             /* 1: hold the buffers temperature sampling needs (dflash_set_sampling);
                                     while the temperature is above 0 the LM heads store fp32 logits */
} dflash_config;

typedef struct {
    int64_t iterations;           /* draft+verify iterations run */
    int64_t tokens;               /* tokens emitted after the prompt, all sequences */
    int64_t accept_hist[DFLASH_MAX_BLOCK];  /* histogram of a (tokens committed - 1) */
    double mean_tau;              /* tokens committed per sequence-iteration */
    double ms_prefill, ms_decode; /* device time of the prefill and decode phases */
    int64_t kernel_launches;      /* kernels this library launched (process-wide counter) */
} dflash_stats;

/* Per-class kernel timing (dflash_profile): launches, summed device time of
 * the launches (CUDA events around each launch on the context's stream) and
 * the algorithmic bytes they move (weights + activations read + outputs
 * written; attention K/V bytes are not counted here). */
typedef struct {
    int64_t launches;
    double ms;
    double bytes;
} dflash_kernel_prof;

/* PROJECTION: every projection launch; ATTENTION: every attention launch;
 * then every projection once more by its shape: GATE_UP (SwiGLU gate/up),
 * QKV, O (attention output), DOWN, LM_HEAD, FUSE (context fuse W_fc),
 * OTHER_PROJ (MoE router).  DRAFT_PASS / VERIFY_PASS: one record per drafter
 * pass (context fuse, drafter layers, head) and per verify pass (target
 * layers, head, accept/commit), events at the pass boundaries only. */
enum {
    DFLASH_PROF_PROJECTION = 0, DFLASH_PROF_ATTENTION = 1, DFLASH_PROF_GATE_UP = 2, DFLASH_PROF_QKV = 3,
    DFLASH_PROF_O = 4, DFLASH_PROF_DOWN = 5, DFLASH_PROF_LM_HEAD = 6, DFLASH_PROF_FUSE = 7,
    DFLASH_PROF_OTHER_PROJ = 8, DFLASH_PROF_DRAFT_PASS = 9, DFLASH_PROF_VERIFY_PASS = 10, DFLASH_PROF_CLASSES = 11
};

/* Bytes of the weight and state arenas for this configuration.
 * Errors: DFLASH_EINVAL on inconsistent configuration, DFLASH_EUNSUPPORTED on
 * shapes the kernels do not implement. */
dflash_status dflash_workspace_size(const dflash_config *cfg, size_t *weight_bytes, size_t *state_bytes);

/* Create a context on the current CUDA device.  weight_arena/state_arena are
 * device pointers (256-byte aligned) of at least the sizes reported above;
 * cuda_stream is a cudaStream_t (NULL = legacy default stream).  Builds the
 * RoPE tables and tensor descriptors; weights may be loaded afterwards. */
dflash_status dflash_create(const dflash_config *cfg, void *weight_arena, size_t weight_bytes,
                            void *state_arena, size_t state_bytes, void *cuda_stream,
                            dflash_ctx **out);

void dflash_destroy(dflash_ctx *ctx);

/* Last error message of the context (owned by ctx, valid until the next call). */
const char *dflash_last_error(const dflash_ctx *ctx);

/* Weight tensors: names, shapes, storage.  Tensors are row-major and live at
 * byte `offset` of the weight arena.  Matrices use cfg.dtype storage (FP8:
 * uint8 codes plus "<name>.scale" [rows] fp32; FP4: packed codes [rows][K/2]
 * (slot type DFLASH_FP4), "<name>.bscale" [K/128][rows][4] (DFLASH_UE8M0) and
 * "<name>.scale"; the embedding stays bf16),
 * RMSNorm gains are always fp32.  Names:
 *   embed [V,H], lm_head [V,H] (both shared by the drafter),
 *   {target|drafter}.L{l}.attn_norm [H], .wqkv [(nq+2nkv)*hd, H] (rows Wq;Wk;Wv),
 *   .wo [H, nq*hd], .ffn_norm [H], .w_gate_up [2F, H] (rows W_gate;W_up),
 *   .w_down [H, F]; MoE layers: .w_router [E,H], .we_gate_up [E,2Fe,H],
 *   .we_down [E,H,Fe]; with qk_norm: .q_norm [hd], .k_norm [hd] (fp32);
 *   {target|drafter}.final_norm [H];
 *   fuse.w_fc [H, n_taps*H], fuse.norm [H]. */
int32_t dflash_weight_count(const dflash_ctx *ctx);
dflash_status dflash_weight_info(const dflash_ctx *ctx, int32_t index, const char **name,
                                 size_t *offset, size_t *numel, int32_t *dtype,
                                 int32_t *ndim, int64_t *shape /* [3] */);
dflash_status dflash_weight_slot(const dflash_ctx *ctx, const char *name, size_t *offset,
                                 size_t *numel, int32_t *dtype);

/* Prefill sequence slot `seq` with prompt[0..n): target causal forward over
 * the prompt (KV cache positions 0..n-1), taps fused into the drafter's
 * context K/V for the same positions, first greedy token returned (it is the
 * anchor of the first block).  Resets the slot.
 * Pages: the prompt pass is not described; it builds what "O alvo sabe mais"
 * (iaemfoco.com DFlash page) needs before the first block -- the target's KV
 * cache and the hidden states of the tapped layers for every prompt position,
 * fused into the context K/V of every drafter layer.
 * Errors: EINVAL (seq out of range, n < 1, ids out of vocab), ECAPACITY
 * (n + block_size > max_len); with first_token: ENUMERIC (non-finite logits,
 * device status word), ETIMEOUT. */
dflash_status dflash_prefill(dflash_ctx *ctx, int32_t seq, const int32_t *prompt, int32_t n,
                             int32_t *first_token);

/* One drafter forward for the listed sequences (seqs[0..n), distinct, each
 * prefilled): block [anchor, mask x (B-1)] at positions p..p+B-1 attends
 * bidirectionally over the context K/V [0, p) and the block itself.
 * Pages: iaemfoco.com DFlash page, "O que o DFlash faz de diferente" (the
 * drafter fills the whole block in one parallel forward) and "O alvo sabe
 * mais" (the context vector of the positions the last verify committed,
 * RMSNorm(W_fc . concat(taps)), is injected into the K/V projections of every
 * drafter layer first); ceviu.com.br page (16 tokens per drafter pass).
 * drafts: host [n*(B-1)] or NULL (then nothing is copied and the call does not
 * synchronise).  Errors: EINVAL, ESTATE, ECAPACITY; with drafts: ENUMERIC,
 * ETIMEOUT. */
dflash_status dflash_draft_block(dflash_ctx *ctx, const int32_t *seqs, int32_t n, int32_t *drafts);

/* Target verify of [anchor, d_1..d_{B-1}] for the same sequences as the last
 * dflash_draft_block (drafts == NULL: use the drafter's; else host [n*(B-1)]
 * supplied by the caller), greedy acceptance a = longest prefix with
 * d_i == g_{i-1}, commit of d_1..d_a and the bonus g_a, KV rollback by length.
 * Pages: iaemfoco.com DFlash page, "O que o DFlash faz de diferente" (the
 * target checks the whole block in one parallel pass) and "Decodificação
 * especulativa tradicional" (accepted tokens are kept; the output equals
 * target-only decoding); imasters.com.br page, "Os três mecanismos por trás do
 * DFlash" (verification in parallel keeps the target's distribution).
 * accept [n], committed [n*B] (first a+1 valid), new_len [n]: host or NULL.
 * Errors: EINVAL, ESTATE (no preceding draft for these sequences); ENUMERIC
 * when a non-finite logit reached an argmax (device status word, sticky until
 * dflash_reset_stats); ETIMEOUT (host wait, or a bounded device wait expired). */
dflash_status dflash_verify_commit(dflash_ctx *ctx, const int32_t *seqs, int32_t n,
                                   const int32_t *drafts, int32_t *accept, int32_t *committed,
                                   int32_t *new_len);

/* Whole generation: prefill each of n prompts into slots 0..n-1, then
 * draft/verify iterations until every sequence holds exactly max_new tokens
 * after its prompt (no EOS).  out: host [n*max_new].  stats: nullable. */
dflash_status dflash_generate(dflash_ctx *ctx, const int32_t *const *prompts, const int32_t *prompt_lens,
                              int32_t n, int32_t max_new, int32_t *out, dflash_stats *stats);

/* Target-only greedy decoding on the same context (slots 0..n-1): prefill,
 * then one target row per step.  Used for speedup baselines and scripts. */
dflash_status dflash_generate_ar(dflash_ctx *ctx, const int32_t *const *prompts, const int32_t *prompt_lens,
                                 int32_t n, int32_t max_new, int32_t *out, double *ms_decode);

/* Enqueue `iters` draft+verify iterations for slots 0..n_seqs-1 (all
 * prefilled) without synchronising: the decode hot loop.  Capacity is checked
 * for the worst case (every iteration commits block_size tokens).
 * Errors: EINVAL, ESTATE, ECAPACITY. */
dflash_status dflash_decode_iters(dflash_ctx *ctx, int32_t n_seqs, int32_t iters);

/* Decode statistics accumulated on the device since the last reset (or the
 * last dflash_generate), plus the process-wide kernel launch counter. */
dflash_status dflash_get_stats(dflash_ctx *ctx, dflash_stats *out);
dflash_status dflash_reset_stats(dflash_ctx *ctx);

/* CUDA-event timing on the context's stream.  mode 0 stops; a nonzero mode
 * starts a fresh record: bit 0 = two events around every projection and
 * attention launch (these break the overlap of consecutive kernels, so the
 * pass is slower while it runs), bit 1 = two events around every drafter and
 * verify pass.  dflash_profile_read fills out[DFLASH_PROF_CLASSES].
 * Errors: EINVAL for a mode outside 0..3. */
dflash_status dflash_profile(dflash_ctx *ctx, int32_t enable);
dflash_status dflash_profile_read(dflash_ctx *ctx, dflash_kernel_prof *out);

/* Draft mode (see DFLASH_DRAFT_SCRIPT); tau in [1, B]. */
dflash_status dflash_set_draft_mode(dflash_ctx *ctx, int32_t mode, int32_t tau);
/* script[i] is the token expected at output index i of slot `seq` (index 0 =
 * first token after the prompt); n <= max_len. */
dflash_status dflash_set_script(dflash_ctx *ctx, int32_t seq, const int32_t *script, int32_t n);

/* Temperature sampling ([P2] iaemfoco.com, "DFlash: Decodificação Especulativa
 * com Blocos em Paralelo ...", "Casos de uso": the method also runs when
 * sampling; [P4] imasters.com.br, "Os três mecanismos por trás do DFlash": the
 * target's distribution is kept).  temperature 0 (the default): greedy.
 * temperature > 0 (needs config.sampling): drafts d_i ~ softmax(z_draft / T),
 * d_i accepted while u * Q_i(d_i) < P_{i-1}(d_i), the first rejected one
 * replaced by a draw from max(0, P_{i-1} - Q_i), a bonus drawn from P_{B-1}
 * when all are accepted; the first token after a prompt and target-only
 * decoding draw from P.  Every draw comes from Philox4x32-10 keyed by seed,
 * with counter (draw index / 4, absolute position, sequence slot, purpose),
 * so runs are reproducible per (seed, slot).  Applies to later calls.
 * Errors: DFLASH_EINVAL for a negative or non-finite temperature;
 * DFLASH_ESTATE without config.sampling or with script drafts. */
dflash_status dflash_set_sampling(dflash_ctx *ctx, double temperature, uint64_t seed);

/* fp32 logits of the last pass (needs keep_logits): which = 0 drafter rows
 * [n_seqs][B][V] (row 0 of each block is the anchor row), 1 verify rows
 * [n_seqs][B][V], 2 last prefill row [V].  host_out sized accordingly;
 * rows_out receives the number of rows copied. */
dflash_status dflash_debug_logits(dflash_ctx *ctx, int32_t which, float *host_out, int64_t capacity,
                                  int64_t *rows_out);

/* Sequence state of slot seq: length (valid target KV positions = position of
 * the anchor), anchor token, tokens emitted after the prompt. */
dflash_status dflash_seq_state(dflash_ctx *ctx, int32_t seq, int32_t *len, int32_t *anchor,
                               int32_t *n_out);

/* Copy the target (which=0) or drafter (which=1) K and V of one layer, sequence
 * and position range [p0, p0+n) to host fp32 buffers [n][n_kv*hd] each. */
dflash_status dflash_debug_kv(dflash_ctx *ctx, int32_t which, int32_t layer, int32_t seq,
                              int32_t p0, int32_t n, float *k_out, float *v_out);

/* Greedy LM-head argmax that uses no caller-provided or allocated scratch.
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot hand the library more device memory at this point -- a serving
 * process that reserved its whole device memory pool up front, or a runtime
 * that forbids cudaMalloc on its decode thread (cudaMalloc can synchronise
 * the device and may fail once the pool is carved up).
 * It recomputes the greedy argmax over the vocabulary of the rows that the
 * last pass on this context fed to the LM head -- which = 0: the drafter rows
 * of the last dflash_draft_block (outputs: n*(B-1) draft ids, as that call
 * returns them); 1: the rows of the last dflash_verify_commit (n*B ids);
 * 2: the last row of the last dflash_prefill (1 id).  The pass named by
 * `which` must be the last one that ran on the context: DFLASH_ESTATE after
 * any other pass (a draft, verify or prefill of another kind, or
 * dflash_generate / dflash_generate_ar / dflash_decode_iters), before any pass,
 * with temperature sampling on, and for which = 0 with script drafts (the
 * ids would not be what the pass returned).  The per-tile
 * partial maxima and the output ids live in one file-scope device array of
 * the library (about 1 MiB; every GPU that loads the library holds it until
 * exit) instead of in the state arena, so the call allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 * Limits: bf16 contexts only (DFLASH_EUNSUPPORTED otherwise); at most 64 rows
 * and a vocabulary of at most 262144 (DFLASH_ECAPACITY beyond).
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the array: calls whose GPU work
 * overlaps (several contexts or streams at once) race on it.  The array keeps
 * the last call's contents; every element a call reads is written by the
 * same call first, so nothing needs clearing.
 * host_out: host buffer of at least *rows_out ids (n*(B-1), n*B or 1);
 * rows_out: receives the number of ids written.  Synchronises the stream.
 * DFLASH_ECUDA if the array's address cannot be looked up or the LM-head
 * projection could not be launched. */
dflash_status dflash_head_argmax_noalloc(dflash_ctx *ctx, int32_t which, int32_t *host_out, int32_t *rows_out);

#ifdef __cplusplus
}
#endif
#endif
